"""Pins of the oracle's FP8 (E4M3, per-tensor scale) pieces, the format of the
shared experts in the Ultra checkpoint recipe, against things other than the
oracle itself: torch's float8_e4m3fn cast (a library routine) on the scaled
values, exact round trips of constructed tensors, the scale's closed form,
saturation, and the shared-expert sum recomputed with torch casts."""
import numpy as np
import pytest
import torch

import lmoe_inputs as LI
from oracle import lmoe_oracle as O


def _torch_e4m3_codes(v32: np.ndarray) -> np.ndarray:
    """torch's E4M3 rounding of fp32 values (in range), as codes."""
    return torch.from_numpy(v32.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_fp8_scale_closed_form():
    rng = np.random.default_rng(1)
    X = rng.standard_normal((64, 48)) * 3.0
    s = O.fp8_scale(X)
    assert s == float(np.float32(np.float32(np.max(np.abs(X))) / np.float32(448.0))) or \
        s == float(np.float32(np.max(np.abs(X)) / 448.0))
    assert O.fp8_scale(np.zeros((4, 4))) == 1.0


def test_fp8_quantize_matches_torch_cast_of_the_scaled_values():
    rng = np.random.default_rng(2)
    X = rng.standard_normal((256, 128)) * np.exp(rng.uniform(-6, 4, size=(256, 128)))
    s = O.fp8_scale(X)
    q = O.fp8_quantize(X, s)
    v = (X / s).astype(np.float32)                 # the fp32 division, as torch sees it
    v = np.clip(v, -448.0, 448.0)                  # amax maps to at most 448 by construction
    assert np.array_equal(q, _torch_e4m3_codes(v))


def test_fp8_quantize_saturates_and_keeps_the_sign():
    q = O.fp8_quantize(np.array([1e6, -1e6, 449.0, -0.0, 0.0]), 1.0)
    assert list(q[:3]) == [0x7E, 0xFE, 0x7E]       # 448 = largest finite E4M3
    assert q[3] == 0x80 and q[4] == 0x00


def test_fp8_exact_round_trip_of_representable_tensors():
    rng = np.random.default_rng(3)
    codes = rng.integers(0, 0x7F, size=(32, 64)).astype(np.uint8) | rng.choice([0, 0x80], size=(32, 64)).astype(np.uint8)
    codes[0, 0] = 0x7E                             # the tensor's amax is 448 * s
    s = 2.0 ** -5                                  # power of two: every step exact
    X = O.e4m3_decode(codes) * s
    assert O.fp8_scale(X) == s
    back = O.fp8_quantize(X, s)
    dec = O.e4m3_decode(back)
    assert np.array_equal(dec, O.e4m3_decode(codes))   # same values (signed zeros aside)
    assert np.array_equal(O.fp8_fake_quant(X, s), X)


def test_shared_experts_fp8_against_torch_casts():
    """The oracle's FP8 shared-expert sum against an independent rendition that
    quantises with torch's float8_e4m3fn casts and sums in fp64."""
    wl = LI.reduced("ultra_nvfp4_fp8shared", T=24, d=128, l=64, N=4, K=2, m=64, n_shared=2, m_shared=96)
    inp = LI.make_inputs(wl)
    x = O.from_bf16_bits(inp["x"])
    ws1 = O.from_bf16_bits(inp["ws1"])
    ws2 = O.from_bf16_bits(inp["ws2"])
    s_x, s_h = inp["shared_x_scale"], inp["shared_h_scale"]
    got, h_codes, (s_w1, s_w2) = O.shared_experts_fp8(x, ws1, ws2, s_x, s_h)

    def tq(v, s):   # torch E4M3 fake quantisation of fp32(v / s), saturated to +-448 first
        t = torch.from_numpy(np.clip((v / s).astype(np.float32), -448.0, 448.0))
        return t.to(torch.float8_e4m3fn).to(torch.float64).numpy() * s

    S, ms, d = ws1.shape
    a_w1 = float(np.float32(np.max(np.abs(ws1)) / 448.0))
    a_w2 = float(np.float32(np.max(np.abs(ws2)) / 448.0))
    assert (s_w1, s_w2) == (a_w1, a_w2)
    xq = tq(x, s_x)
    ref = np.zeros((x.shape[0], d))
    for s in range(S):
        h = np.maximum(xq @ tq(ws1[s], a_w1).T, 0.0) ** 2
        ref += tq(h, s_h) @ tq(ws2[s], a_w2).T
    assert np.allclose(got, ref, rtol=0, atol=1e-12 * np.abs(ref).max())
    assert h_codes.shape == (x.shape[0], S * ms)


def test_forward_with_fp8_shared_experts_adds_their_sum():
    """The layer with FP8 shared experts equals the layer without them plus
    the FP8 shared sum (before the output's BF16 rounding)."""
    wl = LI.reduced("ultra_nvfp4_fp8shared", T=16, d=256, l=256, N=4, K=2, m=256, n_shared=2, m_shared=64)
    inp = LI.make_inputs(wl)
    with_sh = O.forward(wl, inp)
    wl0 = LI.replace(wl, n_shared=0, m_shared=0, shared_fp8=False)
    base = O.forward(wl0, inp)
    ys, _, _ = O.shared_experts_fp8(O.from_bf16_bits(inp["x"]), O.from_bf16_bits(inp["ws1"]),
                                    O.from_bf16_bits(inp["ws2"]), inp["shared_x_scale"], inp["shared_h_scale"])
    assert np.allclose(with_sh["out_unrounded"], base["out_unrounded"] + ys, rtol=0,
                       atol=1e-12 * np.abs(ys).max())
    # and the FP8 sum is close to, but not the same as, the unquantised one
    x = O.from_bf16_bits(inp["x"])
    exact = sum(O.sq_relu(x @ O.from_bf16_bits(inp["ws1"][s]).T) @ O.from_bf16_bits(inp["ws2"][s]).T
                for s in range(2))
    rel = np.sqrt(np.mean((ys - exact) ** 2) / np.mean(exact ** 2))   # E4M3 keeps 3 mantissa bits
    assert 0.005 < rel < 0.15
