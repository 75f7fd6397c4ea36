"""Device failure path without a GPU fault: a bounded pipeline wait that runs
out (an mbarrier nothing arrives on) records LMOE_ERR_DEVICE_TIMEOUT in the
workspace error word and returns; the host reads the status and the context
stays usable for the next layer forward."""
import pytest
import torch

import lmoe_inputs as LI

pytestmark = pytest.mark.gpu

L = pytest.importorskip("latentmoe_fwd_b200")
from gpu_util import DevLayer  # noqa: E402


def test_bounded_wait_runs_out_and_the_context_survives():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    L.selftest_wait_timeout(ws, 20_000_000)          # ~10 ms of SM clock
    st, info = L.read_device_error(ws)
    assert st == L.ERR_DEVICE_TIMEOUT and info == 0x7001
    assert L.read_device_error(ws) == (L.OK, 0)      # reading clears the word
    # the next forward runs normally on the same context
    wl = LI.reduced("ultra_decode", T=40, d=256, l=128, N=16, K=4, m=128)
    dev = DevLayer(wl, LI.make_inputs(wl))
    out = dev.forward()
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()
