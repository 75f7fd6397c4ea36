"""FP8 (E4M3, per-tensor scale) shared experts on the GPU, through the C ABI:
the quantiser bit-exact against the oracle, and layer forwards with FP8 shared
experts against the oracle (which emulates every FP8 rounding point) -- BF16
and NVFP4 routed experts, token-major tiles and the decode (weight-major,
split-K) path, identity and latent projections."""
import numpy as np
import pytest
import torch

import lmoe_inputs as LI
from oracle import lmoe_oracle as O

pytestmark = pytest.mark.gpu

L = pytest.importorskip("latentmoe_fwd_b200")
from gpu_util import fp8_quantize_dev, to_dev  # noqa: E402
from test_gpu_forward import _check_layer  # noqa: E402


@pytest.mark.parametrize("rows,cols", [(1, 16), (37, 256), (512, 1024)])
def test_fp8_quantize_bit_exact_amax_scale(rows, cols):
    rng = np.random.default_rng(rows * 7 + cols)
    v = rng.standard_normal((rows, cols)) * np.exp(rng.uniform(-8, 5, size=(rows, cols)))
    v.reshape(-1)[:: 97] = -0.0                       # signed zeros
    bits = LI.bf16_bits(v)
    x = O.from_bf16_bits(bits)
    codes, scale = fp8_quantize_dev(to_dev(bits, "bf16"), rows, cols)
    s = O.fp8_scale(x)
    assert scale.item() == np.float32(s)
    assert np.array_equal(codes.cpu().numpy(), O.fp8_quantize(x, s))


def test_fp8_quantize_bit_exact_static_scale_with_saturation():
    rng = np.random.default_rng(3)
    v = rng.standard_normal((64, 512)) * 40.0         # some values beyond 448 * s: saturate
    bits = LI.bf16_bits(v)
    x = O.from_bf16_bits(bits)
    s = float(np.float32(0.1234))
    codes, scale = fp8_quantize_dev(to_dev(bits, "bf16"), 64, 512,
                                    scale_in=torch.tensor([s], dtype=torch.float32, device="cuda"))
    assert scale.item() == np.float32(s)
    got = codes.cpu().numpy()
    assert np.array_equal(got, O.fp8_quantize(x, s))
    assert np.any((got & 0x7F) == 0x7E)               # saturated entries present


@pytest.mark.parametrize("T", [16, 48, 300])
def test_forward_bf16_experts_with_fp8_shared_identity(T):
    wl = LI.replace(LI.reduced("std_moe_bf16", T=T, d=512, l=512, N=8, K=2, m=320, n_shared=2, m_shared=256),
                    shared_fp8=True)
    _check_layer(wl, 2e-2)


@pytest.mark.parametrize("T", [32, 700])
def test_forward_bf16_latent_with_fp8_shared(T):
    wl = LI.replace(LI.reduced("ultra_decode", T=T, d=512, l=256, N=64, K=8, m=384, n_shared=2, m_shared=128),
                    shared_fp8=True)
    _check_layer(wl, 2e-2)


@pytest.mark.parametrize("T", [32, 256])
def test_forward_nvfp4_experts_with_fp8_shared(T):
    from test_gpu_nvfp4 import _nvfp4_layer
    wl = LI.reduced("ultra_nvfp4_fp8shared", T=T, d=512, l=256, N=8, K=2, m=256, n_shared=2, m_shared=128)
    _nvfp4_layer(wl)

