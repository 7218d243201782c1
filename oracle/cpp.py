"""ctypes binding of the plain C++ oracle (oracle/nvfp4_oracle.cpp).

TEST INFRASTRUCTURE ONLY: used by tests/, __graft_entry__.smoke() and the CPU
legs of bench.py, never by the product package.  The library is built with
g++ -O2 -ffp-contract=off -fno-fast-math (IEEE binary32/binary64, no fused
multiply-add) on first use, or by ``build()``.  Every function takes and
returns numpy arrays; the arithmetic is all in the C++ file, whose header
lists the readings it follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_DIR = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_DIR, "nvfp4_oracle.cpp")
LIB = os.path.join(_DIR, "liboracle.so")
CXXFLAGS = ["-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-pthread"]

_lib = None


def build(force: bool = False) -> str:
    """Compile liboracle.so when missing or older than its source."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.run(["g++", *CXXFLAGS, SRC, "-o", tmp], check=True)
        os.replace(tmp, LIB)
    return LIB


_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_i32 = ctypes.c_int


class _LayerOut(ctypes.Structure):
    _fields_ = [(n, _vp) for n in ("y", "x_q", "x_sf", "x_s_dec", "offsets", "padded_offsets", "perm",
                                   "inv_perm", "h", "h_q", "h_sf", "h_s_dec", "d")]


_SIGS = {
    "orc_e2m1_encode_n": (None, [_vp, _i64, _vp]),
    "orc_ue4m3_encode_n": (None, [_vp, _i64, _vp]),
    "orc_round_bf16_n": (None, [_vp, _i64, _vp]),
    "orc_e2m1_encode_bits": (None, [ctypes.c_uint32, _i64, _vp, _i32]),
    "orc_ue4m3_encode_bits": (None, [ctypes.c_uint32, _i64, _vp, _i32]),
    "orc_global_scales_n": (None, [_vp, _i64, _vp, _vp]),
    "orc_e2m1_decode": (ctypes.c_double, [ctypes.c_uint8]),
    "orc_ue4m3_decode": (ctypes.c_double, [ctypes.c_uint8]),
    "orc_quantize": (_i32, [_vp, _i64, _i64, _i32, _vp, _vp, _vp, _vp, _vp]),
    "orc_dequantize": (None, [_vp, _vp, _vp, _i64, _i64, _i32, _vp]),
    "orc_route_topk": (_i32, [_vp, _i64, _i32, _i32, _vp, _vp]),
    "orc_permutation": (_i32, [_vp, _i64, _i32, _i32, _vp, _vp, _vp, _vp]),
    "orc_gemm_rows": (None, [_vp, _i64, _vp, _i64, _i64, _vp, _vp, _i32]),
    "orc_grouped_gemm": (None, [_vp, _vp, _i32, _vp, _i64, _i64, _vp, _vp, _i32]),
    "orc_swiglu": (None, [_vp, _i64, _i64, _vp]),
    "orc_combine": (None, [_vp, _i64, _vp, _vp, _i64, _i32, _vp]),
    "orc_swiglu_backward": (None, [_vp, _vp, _vp, _i64, _i64, _vp, _vp]),
    "orc_expert_layer_backward": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i32, _i32, _i32, _vp, _vp,
                                         _vp, _vp]),
    "orc_mxfp8_quantize": (_i32, [_vp, _i64, _i64, _vp, _vp]),
    "orc_mxfp8_dequantize": (None, [_vp, _vp, _i64, _i64, _vp]),
    "orc_expert_layer_w4a8": (_i32, [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i32, _i32, _i32,
                                     ctypes.POINTER(_LayerOut)]),
    "orc_expert_layer_w4a16": (_i32, [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i32, _i32, _i32,
                                      ctypes.POINTER(_LayerOut)]),
    "orc_expert_layer": (_i32, [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i32, _i32, _i32, _i32,
                                ctypes.POINTER(_LayerOut)]),
}


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(LIB)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def threads() -> int:
    return max(1, os.cpu_count() or 1)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


# ------------------------------------------------------------- codecs ----

def e2m1_encode(y) -> np.ndarray:
    y = _c(y, np.float32)
    out = np.empty(y.shape, np.uint8)
    lib().orc_e2m1_encode_n(_p(y), y.size, _p(out))
    return out


def ue4m3_encode(v) -> np.ndarray:
    v = _c(v, np.float32)
    if np.any(v < 0) or np.any(np.isnan(v)):
        raise ValueError("UE4M3 encodes non-negative finite values only")
    out = np.empty(v.shape, np.uint8)
    lib().orc_ue4m3_encode_n(_p(v), v.size, _p(out))
    return out


def e2m1_encode_bits(start: int, n: int) -> np.ndarray:
    """E2M1 codes of the binary32 values with bit patterns start .. start+n-1."""
    out = np.empty(n, np.uint8)
    lib().orc_e2m1_encode_bits(start, n, _p(out), threads())
    return out


def ue4m3_encode_bits(start: int, n: int) -> np.ndarray:
    """UE4M3 codes of the non-negative binary32 values with bit patterns
    start .. start+n-1 (start + n <= 0x7F800000)."""
    if start + n > 0x7F800000:
        raise ValueError("non-negative finite patterns only")
    out = np.empty(n, np.uint8)
    lib().orc_ue4m3_encode_bits(start, n, _p(out), threads())
    return out


def e2m1_decode(codes) -> np.ndarray:
    tab = np.array([lib().orc_e2m1_decode(c) for c in range(16)])
    return tab[np.asarray(codes, dtype=np.uint8) & 0xF]


def ue4m3_decode(codes) -> np.ndarray:
    tab = np.array([lib().orc_ue4m3_decode(c) for c in range(127)])
    return tab[np.asarray(codes, dtype=np.uint8)]


def round_to_bf16(v) -> np.ndarray:
    v = _c(v, np.float64)
    out = np.empty(v.shape, np.float32)
    lib().orc_round_bf16_n(_p(v), v.size, _p(out))
    return out


def global_scales(amax):
    a = _c(np.atleast_1d(amax), np.float32)
    enc = np.empty(a.shape, np.float32)
    dec = np.empty(a.shape, np.float32)
    lib().orc_global_scales_n(_p(a), a.size, _p(enc), _p(dec))
    return enc, dec


# ----------------------------------------------------------- quantize ----

def quantize(x, per_token: bool, amax_in=None) -> dict:
    """Same contract as the numpy oracle's nvfp4.quantize: q [M][K/2],
    sf [M][K/16] row-major, s_dec and amax [1] or [M]."""
    x = _c(x, np.float32)
    M, K = x.shape
    n = M if per_token else 1
    q = np.empty((M, K // 2), np.uint8)
    sf = np.empty((M, K // 16), np.uint8)
    s_dec = np.empty(n, np.float32)
    amax = np.empty(n, np.float32)
    a_in = None if amax_in is None else _c(np.reshape(amax_in, -1), np.float32)
    if a_in is not None and a_in.size != n:
        raise ValueError("amax_in has the wrong size")
    rc = lib().orc_quantize(_p(x), M, K, 1 if per_token else 0, _p(a_in), _p(q), _p(sf), _p(s_dec), _p(amax))
    if rc != 0:
        raise ValueError("K must be a multiple of 16")
    return {"q": q, "sf": sf, "s_dec": s_dec, "amax": amax}


def dequantize(q, sf, s_dec) -> np.ndarray:
    q = _c(q, np.uint8)
    sf = _c(sf, np.uint8)
    s_dec = _c(np.reshape(s_dec, -1), np.float32)
    M, K = q.shape[0], q.shape[1] * 2
    out = np.empty((M, K), np.float64)
    lib().orc_dequantize(_p(q), _p(sf), _p(s_dec), M, K, 1 if s_dec.size == M and M != 1 else 0, _p(out))
    return out


# -------------------------------------------------------------- routing --

def route_topk(logits, k: int):
    logits = _c(logits, np.float32)
    T, E = logits.shape
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    if lib().orc_route_topk(_p(logits), T, E, k, _p(idx), _p(w)) != 0:
        raise ValueError("need 1 <= k <= E")
    return idx, w


def permutation(topk_idx, num_experts: int) -> dict:
    idx = _c(topk_idx, np.int32)
    T, k = idx.shape
    off = np.empty(num_experts + 1, np.int32)
    pad = np.empty(num_experts + 1, np.int32)
    perm = np.empty(T * k, np.int32)
    inv = np.empty(T * k, np.int32)
    if lib().orc_permutation(_p(idx), T, k, num_experts, _p(off), _p(pad), _p(perm), _p(inv)) != 0:
        raise ValueError("expert index out of range")
    return {"offsets": off, "padded_offsets": pad, "perm": perm, "inv_perm": inv.reshape(T, k),
            "counts": np.diff(off).astype(np.int32)}


# ---------------------------------------------------------------- GEMM ----

def gemm_rows(a, w, with_abs: bool = False):
    """out[r][n] = sum_c a[r][c] * w[n][c] (fp64, ascending c); with_abs also
    returns sum_c |a[r][c] * w[n][c]|."""
    a = _c(a, np.float64)
    w = _c(w, np.float64)
    R, K = a.shape
    N = w.shape[0]
    out = np.empty((R, N), np.float64)
    ab = np.empty((R, N), np.float64) if with_abs else None
    lib().orc_gemm_rows(_p(a), R, _p(w), N, K, _p(out), _p(ab), threads())
    return (out, ab) if with_abs else out


def grouped_gemm(a_hat, offsets, w_all, with_abs: bool = False):
    """Rows offsets[e]..offsets[e+1] of a_hat times W_e^T; w_all [E][N][K]."""
    a = _c(a_hat, np.float64)
    w = _c(w_all, np.float64)
    off = _c(offsets, np.int32)
    E, N, K = w.shape
    R = int(off[-1])
    out = np.zeros((R, N), np.float64)
    ab = np.zeros((R, N), np.float64) if with_abs else None
    lib().orc_grouped_gemm(_p(a), _p(off), E, _p(w), N, K, _p(out), _p(ab), threads())
    return (out, ab) if with_abs else out


def swiglu(gu, inter: int) -> np.ndarray:
    gu = _c(gu, np.float64)
    R = gu.shape[0]
    h = np.empty((R, inter), np.float64)
    lib().orc_swiglu(_p(gu), R, inter, _p(h))
    return h


def combine(d_rows_bf16, inv_perm, topk_w) -> np.ndarray:
    d = _c(d_rows_bf16, np.float32)
    inv = _c(inv_perm, np.int32)
    w = _c(topk_w, np.float32)
    T, k = inv.shape
    H = d.shape[1]
    y = np.empty((T, H), np.float32)
    lib().orc_combine(_p(d), H, _p(inv), _p(w), T, k, _p(y))
    return y


def expert_layer(x, topk_idx, topk_w, w_gate_up, w_down, per_token: bool) -> dict:
    """The whole layer (see orc_expert_layer); weights as BF16 values
    w_gate_up [E][2I][H], w_down [E][H][I].  Returns every intermediate."""
    x = _c(x, np.float32)
    idx = _c(topk_idx, np.int32)
    tw = _c(topk_w, np.float32)
    wgu = _c(w_gate_up, np.float32)
    wdn = _c(w_down, np.float32)
    T, H = x.shape
    k = idx.shape[1]
    E, N2, _ = wgu.shape
    I = N2 // 2
    R = T * k
    o = {"y": np.empty((T, H), np.float32), "x_q": np.empty((T, H // 2), np.uint8),
         "x_sf": np.empty((T, H // 16), np.uint8), "x_s_dec": np.empty(T if per_token else 1, np.float32),
         "offsets": np.empty(E + 1, np.int32), "padded_offsets": np.empty(E + 1, np.int32),
         "perm": np.empty(R, np.int32), "inv_perm": np.empty((T, k), np.int32),
         "h": np.empty((R, I), np.float32), "h_q": np.empty((R, I // 2), np.uint8),
         "h_sf": np.empty((R, I // 16), np.uint8), "h_s_dec": np.empty(R if per_token else 1, np.float32),
         "d": np.empty((R, H), np.float32)}
    st = _LayerOut(**{name: arr.ctypes.data for name, arr in o.items()})
    rc = lib().orc_expert_layer(_p(x), _p(idx), _p(tw), _p(wgu), _p(wdn), T, H, I, E, k, 1 if per_token else 0,
                                threads(), ctypes.byref(st))
    if rc != 0:
        raise ValueError("orc_expert_layer: bad shape or routing entry")
    return o


def swiglu_backward(gu, dhp, w):
    """fp64 SwiGLU backward per element: returns dgu [R][2I] and the
    unrounded h [R][I] (see orc_swiglu_backward)."""
    gu = _c(gu, np.float64)
    dhp = _c(dhp, np.float64)
    w = _c(np.reshape(w, -1), np.float64)
    R, I = dhp.shape
    dgu = np.empty((R, 2 * I), np.float64)
    h = np.empty((R, I), np.float64)
    lib().orc_swiglu_backward(_p(gu), _p(dhp), _p(w), R, I, _p(dgu), _p(h))
    return dgu, h


def expert_layer_backward(x, topk_idx, topk_w, w_gate_up, w_down, dy) -> dict:
    """R16: fp64 gradients of sum(dy * y) of the unquantized layer (BF16
    values in): dx [T][H], dw [T][k], dw_gate_up [E][2I][H], dw_down [E][H][I]."""
    x = _c(x, np.float32)
    idx = _c(topk_idx, np.int32)
    tw = _c(topk_w, np.float32)
    wgu = _c(w_gate_up, np.float32)
    wdn = _c(w_down, np.float32)
    dy = _c(dy, np.float32)
    T, H = x.shape
    k = idx.shape[1]
    E, N2, _ = wgu.shape
    I = N2 // 2
    out = {"dx": np.empty((T, H)), "dw": np.empty((T, k)), "dw_gate_up": np.empty((E, 2 * I, H)),
           "dw_down": np.empty((E, H, I))}
    rc = lib().orc_expert_layer_backward(_p(x), _p(idx), _p(tw), _p(wgu), _p(wdn), _p(dy), T, H, I, E, k,
                                         threads(), _p(out["dx"]), _p(out["dw"]), _p(out["dw_gate_up"]),
                                         _p(out["dw_down"]))
    if rc != 0:
        raise ValueError("orc_expert_layer_backward: bad routing entry")
    return out


def mxfp8_quantize(x):
    """R17: MXFP8 codes (E4M3, bit 7 the sign) [M][K] and E8M0 scales [M][K/32]."""
    x = _c(x, np.float32)
    M, K = x.shape
    codes = np.empty((M, K), np.uint8)
    scales = np.empty((M, K // 32), np.uint8)
    if lib().orc_mxfp8_quantize(_p(x), M, K, _p(codes), _p(scales)) != 0:
        raise ValueError("K must be a multiple of 32")
    return codes, scales


def mxfp8_dequantize(codes, scales) -> np.ndarray:
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.uint8)
    M, K = codes.shape
    out = np.empty((M, K), np.float64)
    lib().orc_mxfp8_dequantize(_p(codes), _p(scales), M, K, _p(out))
    return out


def expert_layer_w4a8(x, topk_idx, topk_w, w_gate_up, w_down) -> dict:
    """R20: the layer with NVFP4 weights and MXFP8 activations (x and h).
    Returns y, offsets, perm, inv_perm, h (BF16 before its MXFP8
    requantization, sorted rows) and d."""
    return _layer_variant("orc_expert_layer_w4a8", x, topk_idx, topk_w, w_gate_up, w_down)


def expert_layer_w4a16(x, topk_idx, topk_w, w_gate_up, w_down) -> dict:
    """R19: the layer with BF16 activations and NVFP4 weights (x not
    quantized, h not requantized).  Returns y, offsets, perm, inv_perm, h
    (BF16, sorted rows) and d."""
    return _layer_variant("orc_expert_layer_w4a16", x, topk_idx, topk_w, w_gate_up, w_down)


def _layer_variant(fn, x, topk_idx, topk_w, w_gate_up, w_down) -> dict:
    x = _c(x, np.float32)
    idx = _c(topk_idx, np.int32)
    tw = _c(topk_w, np.float32)
    wgu = _c(w_gate_up, np.float32)
    wdn = _c(w_down, np.float32)
    T, H = x.shape
    k = idx.shape[1]
    E, N2, _ = wgu.shape
    I = N2 // 2
    R = T * k
    o = {"y": np.empty((T, H), np.float32), "offsets": np.empty(E + 1, np.int32),
         "padded_offsets": np.empty(E + 1, np.int32), "perm": np.empty(R, np.int32),
         "inv_perm": np.empty((T, k), np.int32), "h": np.empty((R, I), np.float32), "d": np.empty((R, H), np.float32)}
    fields = {name: arr.ctypes.data for name, arr in o.items()}
    st = _LayerOut(**fields)
    rc = getattr(lib(), fn)(_p(x), _p(idx), _p(tw), _p(wgu), _p(wdn), T, H, I, E, k, threads(), ctypes.byref(st))
    if rc != 0:
        raise ValueError(f"{fn}: bad shape or routing entry")
    return o
