"""Plain, slow CPU oracle for the NVFP4 W4A4 MoE expert layer.

TEST INFRASTRUCTURE ONLY.  This package is imported by ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py``; nothing in the product package may import, call or link
it, and it shares no code, table or helper with the CUDA path.

What it computes follows the miniTE pages (news.hamidun.com "miniTE ... 1.39x
... Qwen3-30B-A3B", list of key facts: native NVFP4 W4A4; www.aib.vote
"miniTE report, NVFP4 RL stability", paragraph 4: the Transformer Engine
token-wise NVFP4 path with contiguous layout, device-side metadata, amax reuse,
grouped matrix multiplication and fusion) plus the public NVFP4 format
definition (E2M1 elements, one E4M3 scale per 16 elements, one FP32 tensor
scale), which the pages name but do not spell out.  Every reading taken where
the pages are silent is listed in the docstring of the function that takes it.

All floating point that decides an integer (a scale code, an element code) is
done in IEEE binary32 with round-to-nearest-even, one operation at a time,
exactly as the quantizer on the GPU must do it; everything else (dequantize,
GEMM, SwiGLU, combine) is fp64.

The oracle the GPU tests compare against is the plain C++ one
(nvfp4_oracle.cpp, built with g++ -O2 -ffp-contract=off -fno-fast-math and
bound by ``cpp``).  The numpy modules are a second, separately written opinion
that the CPU tests check against it bit for bit.

Modules
  cpp      -- ctypes binding of the C++ oracle (codecs, quantize, routing,
              permutation, grouped GEMM, SwiGLU, combine, layer, backward)
  nvfp4    -- E2M1 / UE4M3 codecs, BF16 rounding, quantize, dequantize
  moe      -- routing, permutation, grouped GEMM, SwiGLU + requantize, combine,
              the layer
  backward -- the layer's gradients in the BF16-backward mode
  mxfp8    -- MXFP8 (E4M3 elements, E8M0 block scales) for the W4A8 variant
"""
from . import nvfp4, moe, backward, mxfp8, cpp  # noqa: F401
