"""The failure path of the bounded waits on the GPU: a wait that nothing
completes runs out after its bound, the kernel records the timeout in the
caller's error word and returns, and the context stays usable."""
import time

import pytest
import torch

from nvfp4_moe_grouped_token_b200 import ops

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_reports_timeout():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    ops.wait_selftest(ws)
    assert ops.device_status(ws) == ops.ERR_DEVICE_TIMEOUT
    waited = time.perf_counter() - t0
    assert 1.5 < waited < 60, waited
    # the error word was cleared by the read, and the context still runs work
    assert ops.device_status(ws) == ops.OK
    x = torch.randn(64, 256, device="cuda").to(torch.bfloat16)
    q = torch.empty(64, 128, dtype=torch.uint8, device="cuda")
    sf = torch.empty(64 * 16, dtype=torch.uint8, device="cuda")
    sd = torch.empty(64, dtype=torch.float32, device="cuda")
    ops.nvfp4_quantize(x, q, sf, sd, flags=ops.SCALE_PER_TOKEN)
    torch.cuda.synchronize()
    assert torch.isfinite(sd).all()
