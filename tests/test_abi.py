"""The C-ABI library without a GPU: it loads, exports every function the
header declares, and rejects bad arguments on the host before any launch."""
import ctypes

import pytest

from nvfp4_moe_grouped_token_b200 import ops

L = ops.lib()
P16 = ctypes.c_void_p(1 << 20)          # a fake, 16-byte aligned "device" address
P_ODD = ctypes.c_void_p((1 << 20) + 4)  # misaligned


def test_every_header_function_is_exported():
    names = ops.header_functions()
    assert "moe_expert_layer" in names and "nvfp4_grouped_gemm" in names
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(ops._SIGS), "binding and header disagree"


def test_status_strings_and_version():
    assert L.nvfp4moe_status_string(0) == b"ok"
    for rc in range(-7, 0):
        assert L.nvfp4moe_status_string(rc) != b"unknown status"
    assert L.nvfp4moe_version() >= 100


def test_quantize_rejects_bad_shapes_before_launch():
    q = L.nvfp4_quantize
    assert q(P16, 4, 100, None, P16, P16, P16, P16, 0, None) == -3          # K % 64
    assert q(P16, -1, 64, None, P16, P16, P16, P16, 0, None) == -1
    assert q(P16, 0, 64, None, None, None, None, None, 0, None) == 0          # empty: no-op
    assert q(P_ODD, 4, 64, None, P16, P16, P16, P16, 0, None) == -2
    assert q(P16, 4, 64, None, None, P16, P16, P16, 0, None) == -1           # per tensor needs amax_out
    assert q(None, 4, 64, None, P16, P16, P16, P16, 0, None) == -1


def test_permute_checks():
    assert L.moe_permute(P16, 8, 2, 4, P16, P16, P16, P16, P16, 16, None) == -6   # workspace too small
    assert L.moe_permute(P16, 8, 0, 4, P16, P16, P16, P16, P16, 1 << 20, None) == -1
    assert L.moe_permute(P16, 8, 2, 2000, P16, P16, P16, P16, P16, 1 << 20, None) == -3
    assert L.moe_permute(P16, 8, 40, 4, P16, P16, P16, P16, P16, 1 << 20, None) == -1


def test_route_topk_checks():
    r = L.moe_route_topk
    assert r(P16, 8, 4, 8, P16, P16, None) == -3             # k > E
    assert r(P16, 8, 2000, 8, P16, P16, None) == -3          # E > 1024
    assert r(P16, 8, 128, 40, P16, P16, None) == -3          # k > 32
    assert r(P16, 8, 128, 0, P16, P16, None) == -1
    assert r(P16, -1, 128, 8, P16, P16, None) == -1
    assert r(P16, 0, 128, 8, None, None, None) == 0          # empty: no-op
    assert r(None, 8, 128, 8, P16, P16, None) == -1
    assert r(P_ODD, 8, 128, 8, P16, P16, None) == -2


def test_permute_workspace_size_grows_with_tokens():
    a = ops.moe_permute_workspace_size(128, 8, 128)
    b = ops.moe_permute_workspace_size(129, 8, 128)
    assert 0 < a < b and a % 256 == 0


def test_gemm_checks():
    g = L.nvfp4_grouped_gemm
    args = [P16, P16, P16, P16, P16, P16, P16, P16]
    assert g(*args, 4, 512, 512, 200, P16, None, 0, P16, 256, None) == -3      # K % 256
    assert g(*args, 4, 512, 300, 256, P16, None, 0, P16, 256, None) == -3      # N % 256
    assert g(*args, 4, 500, 512, 256, P16, None, 0, P16, 256, None) == -3      # rows_cap % 128
    assert g(*args, 4, 512, 512, 256, None, None, 0, P16, 256, None) == -1     # no output
    assert g(*args, 4, 512, 512, 256, P16, None, 0, None, 0, None) == -6       # no workspace
    assert g(*args, 0, 512, 512, 256, P16, None, 0, P16, 256, None) == -1


def test_layer_workspace_layout():
    T, H, I, E, k = 16384, 2048, 768, 128, 8
    o = ops.moe_expert_layer_workspace_offsets(T, H, I, E, k)
    assert o["rows_cap"] == ((T * k + 127 * E + 127) // 128) * 128
    names = ["err", "offsets", "padded_offsets", "perm", "inv_perm", "x_q", "x_sf", "x_sdec",
             "h", "h_amax", "h_q", "h_sf", "h_sdec", "d"]
    offs = [o[n] for n in names]
    assert offs == sorted(offs) and all(v % 256 == 0 for v in offs)
    assert o["total"] == ops.moe_expert_layer_workspace_size(T, H, I, E, k)
    cap = o["rows_cap"]
    assert o["x_sf"] - o["x_q"] >= cap * H // 2
    assert o["h_amax"] - o["h"] >= cap * I * 2
    assert o["total"] - o["d"] >= T * k * H * 2


def test_layer_rejects_unsupported_shapes():
    w = ops._Weights(P16.value, P16.value, P16.value, P16.value, 4, 512, 256, ops.W_GATE_UP)
    wd = ops._Weights(P16.value, P16.value, P16.value, P16.value, 4, 256, 256, 0)
    lay = L.moe_expert_layer
    assert lay(P16, P16, P16, ctypes.byref(w), ctypes.byref(wd), 8, 256, 256, 4, 2, P16, 0, P16, 16, None) == -6
    assert lay(P16, P16, P16, ctypes.byref(w), ctypes.byref(wd), 8, 200, 256, 4, 2, P16, 0, P16, 1 << 30, None) == -3
    bad = ops._Weights(P16.value, P16.value, P16.value, P16.value, 4, 512, 256, 0)   # not gate_up ordered
    assert lay(P16, P16, P16, ctypes.byref(bad), ctypes.byref(wd), 8, 256, 256, 4, 2, P16, 0, P16, 1 << 30, None) == -1
    wd2 = ops._Weights(P16.value, P16.value, P16.value, P16.value, 4, 256, 512, 0)  # wrong down K
    assert lay(P16, P16, P16, ctypes.byref(w), ctypes.byref(wd2), 8, 256, 256, 4, 2, P16, 0, P16, 1 << 30, None) == -3


def test_sf_kstep_layout_matches_its_definition():
    import torch
    cap, K = 384, 512
    flat = torch.arange(cap * K // 16, dtype=torch.int64)
    rm = ops.sf_kstep_to_rowmajor(flat, cap, K)
    assert rm.shape == (cap, K // 16)
    assert torch.equal(torch.sort(rm.reshape(-1)).values, flat)
    # byte(row, b) = ((b/16)*rows_cap + row)*16 + b%16, as the header defines it
    for row, b in [(0, 0), (5, 3), (200, 17), (383, 31)]:
        assert int(rm[row, b]) == ((b // 16) * cap + row) * 16 + b % 16


def test_sf_layout_permutation_is_a_bijection():
    import torch
    rows, K = 256, 128
    flat = torch.arange(rows * K // 16, dtype=torch.int64)
    rm = ops.sf_mma_to_rowmajor(flat, rows, K)
    assert rm.shape == (rows, K // 16)
    assert torch.equal(torch.sort(rm.reshape(-1)).values, flat)
    # one known position: row 37, block 5 -> atom 1 of m-tile 0, (37%32)*16 + (37//32)*4 + 1
    assert int(rm[37, 5]) == 1 * 512 + 5 * 16 + 1 * 4 + 1


def test_quantize_permute_checks():
    qp = L.moe_quantize_permute
    a = [P16, P16, P16, P16]                       # topk_idx, inv_perm, offsets, padded_offsets
    assert qp(P16, 8, 100, 2, 4, *a, None, P16, P16, P16, P16, 1024, 0, None) == -3    # K % 64
    assert qp(P16, 8, 256, 40, 4, *a, None, P16, P16, P16, P16, 1024, 0, None) == -1   # k > 32
    assert qp(P16, 0, 256, 2, 4, *a, None, P16, P16, P16, P16, 1024, 0, None) == 0     # empty: no-op
    assert qp(None, 8, 256, 2, 4, *a, None, P16, P16, P16, P16, 1024, 0, None) == -1
    assert qp(P_ODD, 8, 256, 2, 4, *a, None, P16, P16, P16, P16, 1024, 0, None) == -2
    assert qp(P16, 8, 256, 2, 4, *a, None, None, P16, P16, P16, 1024, 0, None) == -1   # per tensor: amax needed


def test_combine_checks():
    c = L.moe_combine
    assert c(P16, P16, P16, 8, 2, 100, P16, None) == -3       # H % 8
    assert c(P16, P16, P16, 8, 0, 256, P16, None) == -1
    assert c(P16, P16, P16, 0, 2, 256, P16, None) == 0        # empty: no-op
    assert c(None, P16, P16, 8, 2, 256, P16, None) == -1
    assert c(P_ODD, P16, P16, 8, 2, 256, P16, None) == -2


def test_prepare_weights_checks():
    pw = L.nvfp4_prepare_weights
    out = ops._Weights(P16.value, P16.value, P16.value, P16.value, 0, 0, 0, 0)
    assert pw(P16, 4, 256, 200, 0, ctypes.byref(out), None) == -3     # K % 256
    assert pw(P16, 4, 300, 256, 0, ctypes.byref(out), None) == -3     # N % 256
    assert pw(None, 4, 256, 256, 0, ctypes.byref(out), None) == -1
    assert pw(P_ODD, 4, 256, 256, 0, ctypes.byref(out), None) == -2
    bad = ops._Weights(None, P16.value, P16.value, P16.value, 0, 0, 0, 0)
    assert pw(P16, 4, 256, 256, 0, ctypes.byref(bad), None) == -1


def test_noalloc_and_diagnostic_checks():
    na = L.moe_permute_noalloc
    assert na(P16, 8, 2, 2000, P16, P16, P16, P16, None) == -3      # E > 1024
    assert na(P16, 8, 40, 4, P16, P16, P16, P16, None) == -1        # k > 32
    assert na(P16, 70000, 2, 4, P16, P16, P16, P16, None) == -6     # beyond the static scratch
    assert L.nvfp4moe_wait_selftest(None, None) == -1
    assert L.nvfp4moe_wait_selftest(P_ODD, None) == -2
    assert L.nvfp4moe_device_status(None, None) == -1


def test_header_compiles_as_c99_and_the_library_links_from_c(tmp_path):
    """The boundary is plain C: a C99 program includes the header, links the
    library and calls entry points that return before any launch."""
    import os
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    lib_dir = os.path.dirname(ops.LIB_PATH)
    src = tmp_path / "abi.c"
    src.write_text(r"""
#include <stdio.h>
#include "nvfp4moe.h"
int main(void) {
  int bad_k = moe_combine((void *)0x100000, (const int32_t *)0x100000, (const float *)0x100000,
                          8, 0, 256, (void *)0x100000, (nvfp4moe_stream_t)0);
  size_t ws = moe_expert_layer_workspace_size(16384, 2048, 768, 128, 8, NVFP4MOE_SCALE_PER_TOKEN);
  printf("%d %s %d %d\n", nvfp4moe_version() >= 100, nvfp4moe_status_string(NVFP4MOE_OK), bad_k, ws > 0);
  return 0;
}
""")
    exe = tmp_path / "abi"
    cc = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(root, "include"), str(src),
                         "-o", str(exe), "-L", lib_dir, "-lnvfp4moe", "-Wl,-rpath," + lib_dir],
                        capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stderr
    assert run.stdout.split() == ["1", "ok", "-1", "1"]
