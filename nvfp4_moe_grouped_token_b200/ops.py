"""Thin Python binding of the nvfp4moe C-ABI (include/nvfp4moe.h).

Argument marshalling only: every function passes torch tensors' device
pointers, sizes and the current CUDA stream to the function of the same name
in libnvfp4moe.so and raises on a non-zero status.  All arithmetic of the path
runs in the library's kernels; torch is used for device memory and streams.
Importing this module fails loudly when the library is missing: there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
import re
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libnvfp4moe.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "nvfp4moe.h")

OK = 0
ERR_CUDA = -4
ERR_DEVICE_TIMEOUT = -5
ERR_DEVICE_CHECK = -7

SCALE_PER_TOKEN = 0x1
STRICT = 0x2
SF_MMA_LAYOUT = 0x4
OUT_PADDED = 0x8
W_GATE_UP = 0x10
KEEP_H = 0x20
BWD_KEEP_DH = 0x40
FAST_COMBINE = 0x80
FUSED_REQUANT = 0x100

_vp, _i64, _i32, _u32, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_uint32, ctypes.c_size_t


class _Weights(ctypes.Structure):
    _fields_ = [("q", _vp), ("sf", _vp), ("s_dec", _vp), ("amax", _vp),
                ("E", _i64), ("N", _i64), ("K", _i64), ("flags", _u32)]


_SIGS = {
    "nvfp4moe_status_string": (ctypes.c_char_p, [_i32]),
    "nvfp4moe_version": (_i32, []),
    "nvfp4moe_device_status": (_i32, [_vp, _vp]),
    "nvfp4moe_wait_selftest": (_i32, [_vp, _vp]),
    "nvfp4_quantize": (_i32, [_vp, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _u32, _vp]),
    "moe_permute_workspace_size": (_sz, [_i64, _i32, _i32]),
    "moe_permute": (_i32, [_vp, _i64, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_permute_noalloc": (_i32, [_vp, _i64, _i32, _i32, _vp, _vp, _vp, _vp, _vp]),
    "moe_route_topk": (_i32, [_vp, _i64, _i32, _i32, _vp, _vp, _vp]),
    "moe_route_permute": (_i32, [_vp, _i64, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_expert_layer_from_logits": (_i32, [_vp, _vp, ctypes.POINTER(_Weights), ctypes.POINTER(_Weights), _i64,
                                            _i64, _i64, _i32, _i32, _vp, _vp, _vp, _u32, _vp, _sz, _vp]),
    "moe_quantize_permute": (_i32, [_vp, _i64, _i64, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp,
                                    _vp, _vp, _vp, _i64, _u32, _vp]),
    "nvfp4_grouped_gemm": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i64, _i64, _i64,
                                  _vp, _vp, _u32, _vp, _sz, _vp]),
    "nvfp4_prepare_weights": (_i32, [_vp, _i64, _i64, _i64, _u32, ctypes.POINTER(_Weights), _vp]),
    "moe_combine": (_i32, [_vp, _vp, _vp, _i64, _i32, _i64, _vp, _vp]),
    "moe_expert_layer_workspace_size": (_sz, [_i64, _i64, _i64, _i32, _i32, _u32]),
    "moe_expert_layer_workspace_offsets": (_i32, [_i64, _i64, _i64, _i32, _i32, _u32,
                                                  ctypes.POINTER(_i64)]),
    "moe_expert_layer": (_i32, [_vp, _vp, _vp, ctypes.POINTER(_Weights), ctypes.POINTER(_Weights),
                                _i64, _i64, _i64, _i32, _i32, _vp, _u32, _vp, _sz, _vp]),
    "moe_expert_layer_profiled": (_i32, [_vp, _vp, _vp, ctypes.POINTER(_Weights),
                                         ctypes.POINTER(_Weights), _i64, _i64, _i64, _i32, _i32,
                                         _vp, _u32, _vp, _sz, _vp, ctypes.POINTER(_vp)]),
    "nvfp4moe_encode_e2m1": (_i32, [_vp, _i64, _vp, _vp]),
    "nvfp4moe_encode_ue4m3": (_i32, [_vp, _i64, _vp, _vp]),
    "nvfp4moe_mma_peak": (_i32, [_i32, _i32, _i32, _vp, _vp, _vp]),
    "moe_expert_layer_backward_workspace_size": (_sz, [_i64, _i64, _i64, _i32, _i32, _u32]),
    "moe_expert_layer_backward_workspace_offsets": (_i32, [_i64, _i64, _i64, _i32, _i32, _u32,
                                                           ctypes.POINTER(_i64)]),
    "moe_expert_layer_backward": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i32, _i32, _vp, _vp,
                                         _vp, _vp, _vp, _vp, _u32, _vp, _sz, _vp]),
    "moe_expert_layer_w4a16_workspace_size": (_sz, [_i64, _i64, _i64, _i32, _i32, _u32]),
    "moe_expert_layer_w4a16_workspace_offsets": (_i32, [_i64, _i64, _i64, _i32, _i32, _u32,
                                                        ctypes.POINTER(_i64)]),
    "moe_expert_layer_w4a16": (_i32, [_vp, _vp, _vp, ctypes.POINTER(_Weights), ctypes.POINTER(_Weights),
                                      _i64, _i64, _i64, _i32, _i32, _vp, _u32, _vp, _sz, _vp]),
    "moe_expert_layer_w4a8_workspace_size": (_sz, [_i64, _i64, _i64, _i32, _i32, _u32]),
    "moe_expert_layer_w4a8_workspace_offsets": (_i32, [_i64, _i64, _i64, _i32, _i32, _u32,
                                                       ctypes.POINTER(_i64)]),
    "moe_expert_layer_w4a8": (_i32, [_vp, _vp, _vp, ctypes.POINTER(_Weights), ctypes.POINTER(_Weights),
                                     _i64, _i64, _i64, _i32, _i32, _vp, _u32, _vp, _sz, _vp]),
    "nvfp4moe_last_cuda_error": (_i32, [ctypes.c_char_p, _sz]),
    "moe_router_logits_workspace_size": (_sz, []),
    "moe_ep_dispatch_workspace_size": (_sz, [_i64, _i32, _i32]),
    "moe_ep_dispatch_pack": (_i32, [_vp, _vp, _i64, _i64, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_ep_rows_cap": (_i64, [_i64, _i32]),
    "moe_ep_arrange_workspace_size": (_sz, [_i32, _i32]),
    "moe_ep_arrange": (_i32, [_vp, _vp, _vp, _vp, _i32, _i32, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _sz,
                              _vp]),
    "moe_ep_experts_workspace_size": (_sz, [_i64, _i64, _i64]),
    "moe_ep_experts": (_i32, [_vp, _vp, _vp, _vp, _vp, _i32, _i64, ctypes.POINTER(_Weights), ctypes.POINTER(_Weights),
                              _i64, _i64, _vp, _vp, _sz, _vp]),
    "moe_ep_return": (_i32, [_vp, _i32, _i32, _i64, _i64, _vp, _vp, _sz, _vp]),
    "moe_router_logits": (_i32, [_vp, _vp, _i64, _i64, _i32, _vp, _vp, _sz, _vp]),
    "nvfp4moe_num_sms": (_i32, []),
}

_LIB = None


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it was not built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m nvfp4_moe_grouped_token_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


def header_functions() -> list[str]:
    """Names of the functions include/nvfp4moe.h declares."""
    text = open(HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b([a-z][a-z0-9_]*)\s*\(", text)) - {"if", "sizeof", "defined"})


class NVFP4Error(RuntimeError):
    pass


def _check(rc: int, what: str):
    if rc != OK:
        msg = lib().nvfp4moe_status_string(rc).decode()
        if rc == ERR_CUDA:
            buf = ctypes.create_string_buffer(256)
            lib().nvfp4moe_last_cuda_error(buf, 256)
            msg += ": " + buf.value.decode()
        raise NVFP4Error(f"{what}: {msg} ({rc})")


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dev(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("tensors must be on a CUDA device")
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


# ------------------------------------------------------------ entry points --

def device_status(workspace: torch.Tensor, stream=None) -> int:
    """nvfp4moe_device_status: synchronizes; returns and clears the error word."""
    return lib().nvfp4moe_device_status(_p(workspace), _stream(stream))


def wait_selftest(workspace: torch.Tensor, stream=None):
    """nvfp4moe_wait_selftest: a kernel whose bounded wait runs out (~2 s)."""
    _dev(workspace)
    _check(lib().nvfp4moe_wait_selftest(_p(workspace), _stream(stream)), "nvfp4moe_wait_selftest")


def nvfp4_quantize(x, q, scales, s_dec, flags=0, amax_in=None, amax_out=None, stream=None):
    _dev(x, q, scales, s_dec, amax_in, amax_out)
    M, K = x.shape
    _check(lib().nvfp4_quantize(_p(x), M, K, _p(amax_in), _p(amax_out), _p(q), _p(scales), _p(s_dec),
                                flags, _stream(stream)), "nvfp4_quantize")


def moe_permute_workspace_size(T, k, E) -> int:
    return int(lib().moe_permute_workspace_size(T, k, E))


def moe_permute(topk_idx, E, offsets, padded_offsets, perm, inv_perm, workspace, stream=None):
    _dev(topk_idx, offsets, padded_offsets, perm, inv_perm, workspace)
    T, k = topk_idx.shape
    _check(lib().moe_permute(_p(topk_idx), T, k, E, _p(offsets), _p(padded_offsets), _p(perm),
                             _p(inv_perm), _p(workspace), workspace.numel() * workspace.element_size(),
                             _stream(stream)), "moe_permute")


def moe_route_topk(logits, k, topk_idx, topk_w, stream=None):
    """moe_route_topk: logits [T][E] FP32 -> topk_idx [T][k] int32, topk_w [T][k] FP32."""
    _dev(logits, topk_idx, topk_w)
    T, E = logits.shape
    _check(lib().moe_route_topk(_p(logits), T, E, k, _p(topk_idx), _p(topk_w), _stream(stream)),
           "moe_route_topk")


def moe_router_logits(x, w_router, logits, workspace=None, stream=None):
    """moe_router_logits: logits [T][E] (FP32, out) = x [T][H] BF16 times
    w_router [E][H] BF16, transposed."""
    if workspace is None:
        workspace = torch.empty(int(lib().moe_router_logits_workspace_size()), dtype=torch.uint8, device=x.device)
    _dev(x, w_router, logits, workspace)
    T, H = x.shape
    E = w_router.shape[0]
    _check(lib().moe_router_logits(_p(x), _p(w_router), T, H, E, _p(logits), _p(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(stream)),
           "moe_router_logits")
    return workspace


# ------------------------------------------------- expert parallelism --
# Argument marshalling for the library's expert-parallel steps; the
# orchestration around the exchanges is in nvfp4_moe_grouped_token_b200.ep.

def _nbytes(t):
    return t.numel() * t.element_size()


def moe_ep_dispatch_pack(x, topk_idx, E, q_send, sf_send, sdec_send, offsets, inv_perm, workspace, stream=None):
    _dev(x, topk_idx, q_send, sf_send, sdec_send, offsets, inv_perm, workspace)
    T, H = x.shape
    k = topk_idx.shape[1]
    _check(lib().moe_ep_dispatch_pack(_p(x), _p(topk_idx), T, H, E, k, _p(q_send), _p(sf_send), _p(sdec_send),
                                      _p(offsets), _p(inv_perm), _p(workspace), _nbytes(workspace), _stream(stream)),
           "moe_ep_dispatch_pack")


def moe_ep_dispatch_workspace_size(T, E, k) -> int:
    return int(lib().moe_ep_dispatch_workspace_size(T, E, k))


def moe_ep_rows_cap(rows_recv, El) -> int:
    return int(lib().moe_ep_rows_cap(rows_recv, El))


def moe_ep_arrange_workspace_size(G, El) -> int:
    return int(lib().moe_ep_arrange_workspace_size(G, El))


def moe_ep_arrange(q_recv, sf_recv, sdec_recv, counts, G, El, H, rows_cap, q_a, sf_a, sdec_a, offsets,
                   padded_offsets, workspace, stream=None):
    _dev(q_recv, sf_recv, sdec_recv, counts, q_a, sf_a, sdec_a, offsets, padded_offsets, workspace)
    rows_recv = q_recv.shape[0]
    _check(lib().moe_ep_arrange(_p(q_recv), _p(sf_recv), _p(sdec_recv), _p(counts), G, El, rows_recv, H, rows_cap,
                                _p(q_a), _p(sf_a), _p(sdec_a), _p(offsets), _p(padded_offsets), _p(workspace),
                                _nbytes(workspace), _stream(stream)), "moe_ep_arrange")


def moe_ep_experts_workspace_size(rows_cap, H, I) -> int:
    return int(lib().moe_ep_experts_workspace_size(rows_cap, H, I))


def moe_ep_experts(q_a, sf_a, sdec_a, offsets, padded_offsets, rows_cap, w_gate_up: "NVFP4Weights",
                   w_down: "NVFP4Weights", d, workspace, stream=None):
    _dev(q_a, sf_a, sdec_a, offsets, padded_offsets, d, workspace)
    gu, dn = w_gate_up.struct(), w_down.struct()
    _check(lib().moe_ep_experts(_p(q_a), _p(sf_a), _p(sdec_a), _p(offsets), _p(padded_offsets), w_down.E, rows_cap,
                                ctypes.byref(gu), ctypes.byref(dn), w_down.N, w_down.K, _p(d), _p(workspace),
                                _nbytes(workspace), _stream(stream)), "moe_ep_experts")


def moe_ep_return(d, G, El, d_send, workspace, stream=None):
    _dev(d, d_send, workspace)
    rows_recv, H = d_send.shape
    _check(lib().moe_ep_return(_p(d), G, El, rows_recv, H, _p(d_send), _p(workspace), _nbytes(workspace),
                               _stream(stream)), "moe_ep_return")


def moe_route_permute(logits, k, topk_idx, topk_w, offsets, padded_offsets, perm, inv_perm, workspace,
                      stream=None):
    """moe_route_permute: router top-k fused with the routing histogram, then
    the permutation; workspace of moe_permute_workspace_size(T, k, E)."""
    _dev(logits, topk_idx, topk_w, offsets, padded_offsets, perm, inv_perm, workspace)
    T, E = logits.shape
    _check(lib().moe_route_permute(_p(logits), T, E, k, _p(topk_idx), _p(topk_w), _p(offsets),
                                   _p(padded_offsets), _p(perm), _p(inv_perm), _p(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(stream)),
           "moe_route_permute")


def moe_permute_noalloc(topk_idx, E, offsets, padded_offsets, perm, inv_perm, stream=None):
    """moe_permute with the library's static scratch: no workspace argument."""
    _dev(topk_idx, offsets, padded_offsets, perm, inv_perm)
    T, k = topk_idx.shape
    _check(lib().moe_permute_noalloc(_p(topk_idx), T, k, E, _p(offsets), _p(padded_offsets), _p(perm),
                                     _p(inv_perm), _stream(stream)), "moe_permute_noalloc")


def moe_quantize_permute(x, topk_idx, inv_perm, offsets, padded_offsets, E, q_rows, sf_rows,
                         s_dec_rows, rows_cap, flags=0, amax_in=None, amax_out=None, stream=None):
    _dev(x, topk_idx, inv_perm, offsets, padded_offsets, q_rows, sf_rows, s_dec_rows, amax_in, amax_out)
    T, K = x.shape
    k = topk_idx.shape[1]
    _check(lib().moe_quantize_permute(_p(x), T, K, k, E, _p(topk_idx), _p(inv_perm), _p(offsets),
                                      _p(padded_offsets), _p(amax_in), _p(amax_out), _p(q_rows),
                                      _p(sf_rows), _p(s_dec_rows), rows_cap, flags, _stream(stream)),
           "moe_quantize_permute")


def nvfp4_grouped_gemm(q_a, sf_a, s_dec_a, weights: "NVFP4Weights", offsets, padded_offsets, rows_cap,
                       out_bf16=None, out_f32=None, flags=0, workspace=None, stream=None):
    _dev(q_a, sf_a, s_dec_a, offsets, padded_offsets, out_bf16, out_f32)
    if workspace is None:
        workspace = torch.zeros(256, dtype=torch.uint8, device=q_a.device)
    w = weights
    _check(lib().nvfp4_grouped_gemm(_p(q_a), _p(sf_a), _p(s_dec_a), _p(w.q), _p(w.sf), _p(w.s_dec),
                                    _p(offsets), _p(padded_offsets), w.E, rows_cap, w.N, w.K,
                                    _p(out_bf16), _p(out_f32), flags, _p(workspace),
                                    workspace.numel(), _stream(stream)), "nvfp4_grouped_gemm")
    return workspace


@dataclass
class NVFP4Weights:
    """Device buffers of one prepared MoE linear (see nvfp4moe_weights)."""
    q: torch.Tensor
    sf: torch.Tensor
    s_dec: torch.Tensor
    amax: torch.Tensor
    E: int
    N: int
    K: int
    flags: int

    def struct(self) -> _Weights:
        return _Weights(self.q.data_ptr(), self.sf.data_ptr(), self.s_dec.data_ptr(),
                        self.amax.data_ptr(), self.E, self.N, self.K, self.flags)

    def experts(self, lo: int, hi: int) -> "NVFP4Weights":
        """Experts [lo, hi) as views of the same buffers (each expert's codes,
        scales and S_dec are its own)."""
        per = self.N * self.K // 16
        return NVFP4Weights(q=self.q[lo:hi], sf=self.sf[lo * per:hi * per], s_dec=self.s_dec[lo:hi],
                            amax=self.amax[lo:hi], E=hi - lo, N=self.N, K=self.K, flags=self.flags)


def nvfp4_prepare_weights(w: torch.Tensor, gate_up: bool, stream=None) -> NVFP4Weights:
    """Quantize BF16 weights [E][N][K] (allocates the outputs with torch)."""
    _dev(w)
    E, N, K = w.shape
    dev = w.device
    out = NVFP4Weights(
        q=torch.empty(E, N, K // 2, dtype=torch.uint8, device=dev),
        sf=torch.empty(E * N * K // 16, dtype=torch.uint8, device=dev),
        s_dec=torch.empty(E, dtype=torch.float32, device=dev),
        amax=torch.empty(E, dtype=torch.float32, device=dev),
        E=E, N=N, K=K, flags=W_GATE_UP if gate_up else 0)
    st = out.struct()
    _check(lib().nvfp4_prepare_weights(_p(w), E, N, K, out.flags, ctypes.byref(st), _stream(stream)),
           "nvfp4_prepare_weights")
    return out


def moe_combine(d, inv_perm, topk_w, y, stream=None):
    _dev(d, inv_perm, topk_w, y)
    T, k = inv_perm.shape
    H = y.shape[1]
    _check(lib().moe_combine(_p(d), _p(inv_perm), _p(topk_w), T, k, H, _p(y), _stream(stream)),
           "moe_combine")


def moe_expert_layer_workspace_size(T, H, I, E, k, flags=0) -> int:
    return int(lib().moe_expert_layer_workspace_size(T, H, I, E, k, flags))


_LAYER_REGIONS = ["err", "offsets", "padded_offsets", "perm", "inv_perm", "x_q", "x_sf", "x_sdec",
                  "h", "h_amax", "h_q", "h_sf", "h_sdec", "d"]


def moe_expert_layer_workspace_offsets(T, H, I, E, k, flags=0) -> dict:
    arr = (ctypes.c_int64 * 16)()
    _check(lib().moe_expert_layer_workspace_offsets(T, H, I, E, k, flags, arr),
           "moe_expert_layer_workspace_offsets")
    out = {name: int(arr[i]) for i, name in enumerate(_LAYER_REGIONS)}
    out["rows_cap"] = int(arr[14])
    out["total"] = int(arr[15])
    return out


def moe_expert_layer(x, topk_idx, topk_w, w_gate_up: NVFP4Weights, w_down: NVFP4Weights, y,
                     workspace, flags=0, stream=None):
    _dev(x, topk_idx, topk_w, y, workspace)
    T, H = x.shape
    k = topk_idx.shape[1]
    I = w_down.K
    gu, dn = w_gate_up.struct(), w_down.struct()
    _check(lib().moe_expert_layer(_p(x), _p(topk_idx), _p(topk_w), ctypes.byref(gu), ctypes.byref(dn),
                                  T, H, I, w_down.E, k, _p(y), flags, _p(workspace),
                                  workspace.numel() * workspace.element_size(), _stream(stream)),
           "moe_expert_layer")


def moe_expert_layer_from_logits(x, logits, w_gate_up: NVFP4Weights, w_down: NVFP4Weights, topk_idx, topk_w,
                                 y, workspace, flags=0, stream=None):
    """moe_expert_layer_from_logits: the layer routed from router logits
    inside its histogram kernel; topk_idx / topk_w are written."""
    _dev(x, logits, topk_idx, topk_w, y, workspace)
    T, H = x.shape
    k = topk_idx.shape[1]
    I = w_down.K
    gu, dn = w_gate_up.struct(), w_down.struct()
    _check(lib().moe_expert_layer_from_logits(_p(x), _p(logits), ctypes.byref(gu), ctypes.byref(dn), T, H, I,
                                              w_down.E, k, _p(topk_idx), _p(topk_w), _p(y), flags, _p(workspace),
                                              workspace.numel() * workspace.element_size(), _stream(stream)),
           "moe_expert_layer_from_logits")


STAGES = ["route", "quantize_permute", "gate_up_swiglu", "requant_h", "down", "combine"]


def moe_expert_layer_profiled(x, topk_idx, topk_w, w_gate_up: NVFP4Weights, w_down: NVFP4Weights, y,
                              workspace, events, flags=0, stream=None):
    """moe_expert_layer recording the 7 torch.cuda.Event objects in `events`
    (created with enable_timing=True) at the stage boundaries; a None entry
    records nothing there."""
    _dev(x, topk_idx, topk_w, y, workspace)
    T, H = x.shape
    k = topk_idx.shape[1]
    I = w_down.K
    arr = (ctypes.c_void_p * 7)()
    for i, ev in enumerate(events):
        arr[i] = None if ev is None else ctypes.c_void_p(ev.cuda_event)
    gu, dn = w_gate_up.struct(), w_down.struct()
    _check(lib().moe_expert_layer_profiled(_p(x), _p(topk_idx), _p(topk_w), ctypes.byref(gu),
                                           ctypes.byref(dn), T, H, I, w_down.E, k, _p(y), flags,
                                           _p(workspace), workspace.numel() * workspace.element_size(),
                                           _stream(stream), arr), "moe_expert_layer_profiled")


# ------------------------------------------------------------- backward --

def moe_expert_layer_backward_workspace_size(T, H, I, E, k, flags=0) -> int:
    return int(lib().moe_expert_layer_backward_workspace_size(T, H, I, E, k, flags))


_BWD_REGIONS = ["err", "offsets", "padded_offsets", "perm", "inv_perm", "x_rows", "dy_rows", "w_rows", "g",
                "dg", "hw", "dw_part", "dx_rows", "dh"]


def moe_expert_layer_backward_workspace_offsets(T, H, I, E, k, flags=0) -> dict:
    arr = (ctypes.c_int64 * 16)()
    _check(lib().moe_expert_layer_backward_workspace_offsets(T, H, I, E, k, flags, arr),
           "moe_expert_layer_backward_workspace_offsets")
    out = {name: int(arr[i]) for i, name in enumerate(_BWD_REGIONS)}
    out["rows_cap"] = int(arr[14])
    out["total"] = int(arr[15])
    return out


def moe_expert_layer_backward(x, topk_idx, topk_w, w_gate_up, w_down, dy, dx, d_topk_w, workspace,
                              dw_gate_up_bf16=None, dw_gate_up_f32=None, dw_down_bf16=None, dw_down_f32=None,
                              flags=0, stream=None):
    """Backward of the layer in the BF16-backward mode (moe_expert_layer_backward):
    w_gate_up [E][2I][H] and w_down [E][H][I] are the BF16 weights."""
    _dev(x, topk_idx, topk_w, w_gate_up, w_down, dy, dx, d_topk_w, workspace, dw_gate_up_bf16, dw_gate_up_f32,
         dw_down_bf16, dw_down_f32)
    T, H = x.shape
    k = topk_idx.shape[1]
    E, N2, _ = w_gate_up.shape
    _check(lib().moe_expert_layer_backward(_p(x), _p(topk_idx), _p(topk_w), _p(w_gate_up), _p(w_down), _p(dy), T,
                                           H, N2 // 2, E, k, _p(dx), _p(d_topk_w), _p(dw_gate_up_bf16),
                                           _p(dw_gate_up_f32), _p(dw_down_bf16), _p(dw_down_f32), flags,
                                           _p(workspace), workspace.numel() * workspace.element_size(),
                                           _stream(stream)), "moe_expert_layer_backward")


def backward_views(workspace: torch.Tensor, T, H, I, E, k, flags=0) -> dict:
    """Typed views of the backward workspace's regions (for inspection in tests)."""
    o = moe_expert_layer_backward_workspace_offsets(T, H, I, E, k, flags)
    cap = o["rows_cap"]
    R = T * k
    ws = workspace

    def view(name, nbytes, dtype, shape):
        return ws[o[name]:o[name] + nbytes].view(dtype).view(*shape)

    v = {
        "rows_cap": cap,
        "offsets": view("offsets", (E + 1) * 4, torch.int32, (E + 1,)),
        "padded_offsets": view("padded_offsets", (E + 1) * 4, torch.int32, (E + 1,)),
        "perm": view("perm", R * 4, torch.int32, (R,)),
        "inv_perm": view("inv_perm", R * 4, torch.int32, (T, k)),
        "x_rows": view("x_rows", cap * H * 2, torch.bfloat16, (cap, H)),
        "dy_rows": view("dy_rows", cap * H * 2, torch.bfloat16, (cap, H)),
        "w_rows": view("w_rows", cap * 4, torch.float32, (cap,)),
        "g": view("g", cap * 2 * I * 2, torch.bfloat16, (cap, 2 * I)),
        "dg": view("dg", cap * 2 * I * 2, torch.bfloat16, (cap, 2 * I)),
        "hw": view("hw", cap * I * 2, torch.bfloat16, (cap, I)),
        "dw_part": view("dw_part", cap * (I // 128) * 4, torch.float32, (cap, I // 128)),
        "dx_rows": view("dx_rows", R * H * 2, torch.bfloat16, (R, H)),
    }
    if flags & BWD_KEEP_DH:
        v["dh"] = view("dh", cap * I * 4, torch.float32, (cap, I))
    return v


# ---------------------------------------------------------------- W4A16 --

def moe_expert_layer_w4a16_workspace_size(T, H, I, E, k, flags=0) -> int:
    return int(lib().moe_expert_layer_w4a16_workspace_size(T, H, I, E, k, flags))


def moe_expert_layer_w4a8_workspace_size(T, H, I, E, k, flags=0) -> int:
    return int(lib().moe_expert_layer_w4a8_workspace_size(T, H, I, E, k, flags))


_W4AX_REGIONS = ["err", "offsets", "padded_offsets", "perm", "inv_perm", "x_rows", "h", "d", "h_pre"]


def _w4ax_offsets(fn, T, H, I, E, k, flags) -> dict:
    arr = (ctypes.c_int64 * 16)()
    _check(getattr(lib(), fn)(T, H, I, E, k, flags, arr), fn)
    out = {name: int(arr[i]) for i, name in enumerate(_W4AX_REGIONS)}
    out["rows_cap"] = int(arr[14])
    out["total"] = int(arr[15])
    return out


def moe_expert_layer_w4a16_workspace_offsets(T, H, I, E, k, flags=0) -> dict:
    return _w4ax_offsets("moe_expert_layer_w4a16_workspace_offsets", T, H, I, E, k, flags)


def moe_expert_layer_w4a8_workspace_offsets(T, H, I, E, k, flags=0) -> dict:
    return _w4ax_offsets("moe_expert_layer_w4a8_workspace_offsets", T, H, I, E, k, flags)


def _w4ax_layer(fn, x, topk_idx, topk_w, w_gate_up, w_down, y, workspace, flags, stream):
    _dev(x, topk_idx, topk_w, y, workspace)
    T, H = x.shape
    k = topk_idx.shape[1]
    I = w_down.K
    gu, dn = w_gate_up.struct(), w_down.struct()
    _check(getattr(lib(), fn)(_p(x), _p(topk_idx), _p(topk_w), ctypes.byref(gu), ctypes.byref(dn), T, H, I,
                              w_down.E, k, _p(y), flags, _p(workspace), workspace.numel() * workspace.element_size(),
                              _stream(stream)), fn)


def moe_expert_layer_w4a16(x, topk_idx, topk_w, w_gate_up: NVFP4Weights, w_down: NVFP4Weights, y,
                           workspace, flags=0, stream=None):
    """moe_expert_layer_w4a16: BF16 activations, the same prepared NVFP4
    weights as moe_expert_layer."""
    _w4ax_layer("moe_expert_layer_w4a16", x, topk_idx, topk_w, w_gate_up, w_down, y, workspace, flags, stream)


def moe_expert_layer_w4a8(x, topk_idx, topk_w, w_gate_up: NVFP4Weights, w_down: NVFP4Weights, y,
                          workspace, flags=0, stream=None):
    """moe_expert_layer_w4a8: MXFP8 activations (x and h), the same prepared
    NVFP4 weights as moe_expert_layer; flags 0 or KEEP_H."""
    _w4ax_layer("moe_expert_layer_w4a8", x, topk_idx, topk_w, w_gate_up, w_down, y, workspace, flags, stream)


def w4a16_views(workspace: torch.Tensor, T, H, I, E, k, flags=0, w4a8=False) -> dict:
    """Typed views of the W4A16 / W4A8 workspace's regions (for inspection in tests)."""
    o = (moe_expert_layer_w4a8_workspace_offsets if w4a8 else moe_expert_layer_w4a16_workspace_offsets)(
        T, H, I, E, k, flags)
    cap = o["rows_cap"]
    R = T * k
    ws = workspace

    def view(name, nbytes, dtype, shape):
        return ws[o[name]:o[name] + nbytes].view(dtype).view(*shape)

    v = {
        "rows_cap": cap,
        "offsets": view("offsets", (E + 1) * 4, torch.int32, (E + 1,)),
        "padded_offsets": view("padded_offsets", (E + 1) * 4, torch.int32, (E + 1,)),
        "perm": view("perm", R * 4, torch.int32, (R,)),
        "inv_perm": view("inv_perm", R * 4, torch.int32, (T, k)),
        "x_rows": view("x_rows", cap * H * 2, torch.bfloat16, (cap, H)),
        "h": view("h", cap * I * 2, torch.bfloat16, (cap, I)),
        "d": view("d", R * H * 2, torch.bfloat16, (R, H)),
    }
    if w4a8 and flags & KEEP_H:
        v["h_pre"] = view("h_pre", cap * I * 2, torch.bfloat16, (cap, I))
    return v


def nvfp4moe_encode_e2m1(y: torch.Tensor, codes: torch.Tensor, stream=None):
    _dev(y, codes)
    _check(lib().nvfp4moe_encode_e2m1(_p(y), y.numel(), _p(codes), _stream(stream)), "encode_e2m1")


def nvfp4moe_encode_ue4m3(v: torch.Tensor, codes: torch.Tensor, stream=None):
    _dev(v, codes)
    _check(lib().nvfp4moe_encode_ue4m3(_p(v), v.numel(), _p(codes), _stream(stream)), "encode_ue4m3")


def mma_peak(iters: int = 4000, scale_writes: bool = True, grid: int = 0, stream=None) -> dict:
    """nvfp4moe_mma_peak: dense block-scaled FP4 MMA throughput on this GPU,
    timed with CUDA events on the launching stream.  Returns TFLOP/s and FLOP
    per SM per cycle."""
    grid = grid or lib().nvfp4moe_num_sms()
    cyc = torch.zeros(grid, dtype=torch.int64, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    s = torch.cuda.current_stream() if stream is None else stream
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    _check(lib().nvfp4moe_mma_peak(iters, 1 if scale_writes else 0, grid, _p(cyc), _p(ws), _stream(s)),
           "nvfp4moe_mma_peak")
    e1.record(s)
    torch.cuda.synchronize()
    if device_status(ws) != OK:
        raise NVFP4Error("mma peak probe wait timed out")
    flop = grid * iters * 4 * 2.0 * 128 * 256 * 64
    ms = e0.elapsed_time(e1)
    c = cyc.float().mean().item()
    return {"tflops": flop / (ms * 1e-3) / 1e12, "flop_per_sm_cycle": flop / grid / c, "ms": ms,
            "cycles_mean": c, "grid": grid, "iters": iters, "scale_writes": bool(scale_writes)}


# ------------------------------------------------------------------ helpers --

def layer_views(workspace: torch.Tensor, T, H, I, E, k, flags=0) -> dict:
    """Typed views of the layer workspace's regions (for inspection in tests)."""
    o = moe_expert_layer_workspace_offsets(T, H, I, E, k, flags)
    cap = o["rows_cap"]
    R = T * k
    ws = workspace

    def view(name, nbytes, dtype, shape):
        return ws[o[name]:o[name] + nbytes].view(dtype).view(*shape)

    return {
        "rows_cap": cap,
        "offsets": view("offsets", (E + 1) * 4, torch.int32, (E + 1,)),
        "padded_offsets": view("padded_offsets", (E + 1) * 4, torch.int32, (E + 1,)),
        "perm": view("perm", R * 4, torch.int32, (R,)),
        "inv_perm": view("inv_perm", R * 4, torch.int32, (T, k)),
        "x_q": view("x_q", cap * H // 2, torch.uint8, (cap, H // 2)),
        "x_sf": view("x_sf", cap * H // 16, torch.uint8, (cap * H // 16,)),
        "x_sdec": view("x_sdec", cap * 4, torch.float32, (cap,)),
        "h": view("h", cap * I * 2, torch.bfloat16, (cap, I)),
        "h_amax": view("h_amax", cap * 4, torch.float32, (cap,)),
        "h_q": view("h_q", cap * I // 2, torch.uint8, (cap, I // 2)),
        "h_sf": view("h_sf", cap * I // 16, torch.uint8, (cap * I // 16,)),
        "h_sdec": view("h_sdec", cap * 4, torch.float32, (cap,)),
        "d": view("d", R * H * 2, torch.bfloat16, (R, H)),
        "header_f32": ws[0:256].view(torch.float32),
    }


def sf_kstep_to_rowmajor(sf_flat: torch.Tensor, rows_cap: int, K: int) -> torch.Tensor:
    """Rearrange scales stored in the K-step-major layout of the padded grouped
    layout ([K/256][rows_cap][16]) into row-major [rows_cap][K/16]."""
    a = sf_flat[: rows_cap * (K // 16)].view(K // 256, rows_cap, 16)
    return a.permute(1, 0, 2).reshape(rows_cap, K // 16)


def sf_mma_to_rowmajor(sf_flat: torch.Tensor, rows: int, K: int) -> torch.Tensor:
    """Rearrange scales stored in the MMA atom layout into row-major
    [rows][K/16] (an index permutation; used to compare layouts in tests)."""
    rows_pad = (rows + 127) // 128 * 128
    nb = K // 16
    a = sf_flat[: rows_pad * nb].view(rows_pad // 128, K // 64, 32, 4, 4)  # [mt][kat][r%32][r/32%4][b%4]
    a = a.permute(0, 3, 2, 1, 4).reshape(rows_pad, nb)                     # row = mt*128 + q*32 + r
    return a[:rows]
