"""lmoe_forward captured in a CUDA graph and replayed: the replay equals the
eager call bit for bit, also after new inputs are copied into the captured
buffers. The cases take every dispatch path of the forward: BF16 latent
prefill (top-K and permutation on a side stream beside the down-projection,
forked and joined inside the capture), NVFP4 experts, decode sizes (split-K
projections) and identity projections with shared experts."""
import pytest
import torch

import lmoe_inputs as LI

pytestmark = pytest.mark.gpu

L = pytest.importorskip("latentmoe_fwd_b200")
from gpu_util import DevLayer, to_dev  # noqa: E402

CASES = {
    "latent_prefill": ("ultra_zipf", dict(T=900, d=1024, l=512, N=32, K=6, m=512)),
    "nvfp4_prefill": ("ultra_nvfp4", dict(T=700, d=1024, l=512, N=32, K=6, m=512)),
    "latent_decode": ("ultra_decode", dict(T=32, d=1024, l=512, N=64, K=6, m=256)),
    "identity_shared": ("std_moe_bf16", dict(T=300, d=256, l=256, N=16, K=4, m=256, n_shared=2, m_shared=128)),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_forward_replays_from_a_cuda_graph(case):
    name, shape = CASES[case]
    wl = LI.reduced(name, **shape)
    dev = DevLayer(wl, LI.make_inputs(wl))
    ws = L.workspace(dev.cfg, L.OP_FORWARD)
    shape_out = (wl.T, wl.d)
    eager = torch.empty(shape_out, dtype=dev.x.dtype, device="cuda")
    L.forward(dev.cfg, dev.w, dev.x, eager, ws)
    torch.cuda.synchronize()

    s = torch.cuda.Stream()
    out = torch.zeros(shape_out, dtype=dev.x.dtype, device="cuda")
    with torch.cuda.stream(s):   # first use on this thread and stream before the capture
        L.forward(dev.cfg, dev.w, dev.x, out, ws, stream=s)
    torch.cuda.synchronize()
    out.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        L.forward(dev.cfg, dev.w, dev.x, out, ws, stream=s)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager)

    # new inputs in the captured buffer: the replay follows them
    wl2 = LI.replace(wl, seed=wl.seed + 1)
    x2 = to_dev(LI.make_inputs(wl2)["x"], dev.st)
    dev.x.copy_(x2)
    g.replay()
    eager2 = torch.empty_like(eager)
    L.forward(dev.cfg, dev.w, dev.x, eager2, ws)
    torch.cuda.synchronize()
    assert torch.equal(out, eager2)
    st, info = L.read_device_error(ws)
    assert st == L.OK, (L.status_string(st), hex(info))
