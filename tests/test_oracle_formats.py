"""Pins for the oracle's number formats: BF16/fp32 rounding points and the
NVFP4 element (E2M1) and block-scale (E4M3) formats named on the greeksharifa
page, section 2.4 "NVFP4 Training" (E2M1 elements, 16-element micro-blocks,
E4M3 block scales, an FP32 global scale).

Each pin is independent of the code it checks: a closed-form value table
(tests/golden), a library cast (torch bfloat16 / float8_e4m3fn), brute-force
nearest-value search, or exactly representable constructed tensors.
"""
import os

import numpy as np
import pytest
import torch

from oracle import lmoe_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_table(name):
    vals = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                code, val = line.split()
                vals.append((int(code, 0), float(val)))
    return vals


def test_e2m1_table_matches_golden():
    for code, val in _golden_table("e2m1_codes.txt"):
        got = O.e2m1_decode(code)
        assert got == val and np.signbit(got) == np.signbit(val), (code, got, val)


def test_e4m3_selected_values_match_golden():
    for code, val in _golden_table("e4m3_codes.txt"):
        got = O.e4m3_decode(code)
        if np.isnan(val):
            assert np.isnan(got)
        else:
            assert got == val, (code, got, val)


def test_e4m3_decode_matches_torch_for_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = O.e4m3_decode(codes)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(1)
    # log-uniform magnitudes over the whole finite range, plus every midpoint
    v = np.exp(rng.uniform(np.log(2.0 ** -12), np.log(448.0), 200000)).astype(np.float32)
    mids = ((O.E4M3_MAG[1:] + O.E4M3_MAG[:-1]) / 2).astype(np.float32)
    v = np.concatenate([v, mids, O.E4M3_MAG.astype(np.float32)])
    v = np.concatenate([v, -v])
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = O.e4m3_encode(v.astype(np.float64))
    assert np.array_equal(got, ref)


def test_e4m3_encode_saturates():
    assert O.e4m3_decode(O.e4m3_encode(1e6)) == 448.0
    assert O.e4m3_decode(O.e4m3_encode(449.0)) == 448.0
    assert O.e4m3_encode(0.0) == 0


def _brute_e2m1(v):
    """Nearest E2M1 magnitude by scanning all 8 codes; ties to the even code."""
    best = None
    for c in range(8):
        dist = abs(abs(v) - O.E2M1_MAG[c])
        if best is None or dist < best[0] or (dist == best[0] and c % 2 == 0):
            best = (dist, c)
    c = best[1] if abs(v) <= 6.0 else 7
    return c | (8 if np.signbit(v) else 0)


def test_e2m1_encode_brute_force():
    rng = np.random.default_rng(2)
    v = np.concatenate([rng.uniform(-8, 8, 5000),
                        np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 7.0, 0.0, -0.0]),
                        -np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])])
    got = O.e2m1_encode(v)
    ref = np.array([_brute_e2m1(t) for t in v], dtype=np.uint8)
    assert np.array_equal(got, ref)


def test_e2m1_ties_to_even_values():
    ties = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    for v, want in ties.items():
        assert O.e2m1_decode(O.e2m1_encode(v)) == want
        assert O.e2m1_decode(O.e2m1_encode(-v)) == -want


def test_round_bf16_matches_torch_on_fp32_inputs():
    rng = np.random.default_rng(3)
    f = (rng.standard_normal(100000) * np.exp(rng.uniform(-30, 30, 100000))).astype(np.float32)
    tiny = (rng.standard_normal(2000) * 2.0 ** -130).astype(np.float32)   # bf16 subnormals
    f = np.concatenate([f, tiny])
    ref = torch.from_numpy(f).to(torch.bfloat16).to(torch.float64).numpy()
    got = O.round_bf16(f.astype(np.float64))
    assert np.array_equal(got, ref)


def test_round_bf16_ties_and_fp64_inputs():
    one = 1.0
    ulp = 2.0 ** -7
    assert O.round_bf16(one + ulp / 2) == one                 # tie -> even (1.0)
    assert O.round_bf16(one + 3 * ulp / 2) == one + 2 * ulp   # tie -> even
    assert O.round_bf16(one + ulp / 2 + 2.0 ** -40) == one + ulp  # just above the tie
    # an fp64 value whose fp32 rounding would land on the tie: direct rounding is used
    v = one + ulp / 2 - 2.0 ** -30
    assert O.round_bf16(v) == one


def test_round_f32_is_ieee_cast():
    rng = np.random.default_rng(4)
    v = rng.standard_normal(1000) * 1e3
    assert np.array_equal(O.round_f32(v), torch.from_numpy(v).float().double().numpy())


def _exact_block_tensor(rng, rows, nblk, s_g):
    """Blocks whose largest entry is 6*s_b*s_g and every entry a grid point,
    with power-of-two s_g and s_b, so every fp32 step of the recipe is exact."""
    X = np.zeros((rows, nblk * 16))
    sbs = 2.0 ** rng.integers(-6, 9, size=(rows, nblk))   # E4M3 normals, <= 256
    sbs[0, 0] = 448.0 if s_g == 1.0 else sbs[0, 0]
    for r in range(rows):
        for b in range(nblk):
            q = rng.choice(O.E2M1_MAG, 16) * rng.choice([-1.0, 1.0], 16)
            q[rng.integers(16)] = 6.0 * rng.choice([-1.0, 1.0])
            X[r, b * 16:(b + 1) * 16] = q * sbs[r, b] * s_g
    return X


@pytest.mark.parametrize("s_g", [1.0, 2.0 ** -3, 2.0 ** 5])
def test_nvfp4_round_trip_exact(s_g):
    rng = np.random.default_rng(5)
    X = _exact_block_tensor(rng, 8, 4, s_g)
    codes, sf, g = O.nvfp4_quantize(X, s_g)
    assert g == s_g
    assert np.array_equal(O.nvfp4_dequantize(codes, sf, g), X)


def test_nvfp4_global_scale_current_amax():
    rng = np.random.default_rng(6)
    X = O.round_bf16(rng.standard_normal((4, 64)))
    amax = np.max(np.abs(X))
    assert O.nvfp4_global_scale(X) == np.float32(np.float32(amax) / np.float32(2688.0))
    assert O.nvfp4_global_scale(np.zeros((2, 16))) == 1.0


def test_nvfp4_codes_are_nearest_grid_points():
    """Each element's code is the brute-force nearest E2M1 point of x / (s_b*s_g),
    the block scale is the E4M3 rounding of amax_b / (6 s_g), and the block
    max never exceeds the grid (|x_hat| <= 6 * s_b * s_g)."""
    rng = np.random.default_rng(7)
    X = O.round_bf16(rng.standard_normal((6, 96)) * np.exp(rng.uniform(-4, 4, (6, 1))))
    codes, sf, s_g = O.nvfp4_quantize(X)
    q = O.nvfp4_unpack(codes)
    for r in range(X.shape[0]):
        for b in range(X.shape[1] // 16):
            blk = X[r, b * 16:(b + 1) * 16]
            amax = np.float32(np.max(np.abs(blk)))
            r_f32 = np.float32(amax / np.float32(np.float32(s_g) * np.float32(6.0)))
            assert sf[r, b] == torch.tensor([float(r_f32)]).to(torch.float8_e4m3fn).view(torch.uint8).item()
            sb = O.e4m3_decode(sf[r, b])
            sc = np.float32(np.float32(sb) * np.float32(s_g))
            for i in range(16):
                v = float(np.float32(np.float32(blk[i]) / sc)) if sb != 0 else 0.0
                want = _brute_e2m1(v) if sb != 0 else 0
                assert q[r, b * 16 + i] == want
    deq = O.nvfp4_dequantize(codes, sf, s_g)
    assert np.all(np.abs(deq) <= 6 * np.repeat(O.e4m3_decode(sf), 16, axis=1) * s_g)
    # half a grid step of error at most, relative to the block scale
    err = np.abs(deq - X) / (np.repeat(O.e4m3_decode(sf), 16, axis=1) * s_g)
    assert np.all(err <= 1.0 + 1e-12)


def test_nvfp4_packing_low_nibble_first():
    X = np.zeros((1, 16))
    X[0, 0] = 6.0
    X[0, 1] = -0.5
    codes, sf, s_g = O.nvfp4_quantize(X, 1.0)
    # block amax 6 -> s_b = E4M3(6 / 6) = 1.0
    assert O.e4m3_decode(sf[0, 0]) == 1.0
    assert codes[0, 0] == (0x7 | (0x9 << 4))


def test_nvfp4_zero_scale_block_is_all_zero_codes():
    X = np.zeros((1, 32))
    X[0, 16] = 1.0
    X[0, 3] = -1e-30    # rounds the block scale to 0
    codes, sf, s_g = O.nvfp4_quantize(X)
    assert sf[0, 0] == 0
    assert np.all(O.nvfp4_unpack(codes)[0, :16] == 0)


# ---- two-dimensional (16 x 16) weight blocks ----

def test_nvfp4_2d_transpose_symmetry():
    """16 x 16 blocks quantise W and W^T alike: codes and scales transpose."""
    rng = np.random.default_rng(11)
    W = O.round_bf16(rng.standard_normal((48, 64)) * np.exp(rng.uniform(-3, 3, (48, 1))))
    c, sf, g = O.nvfp4_quantize_2d(W)
    ct, sft, gt = O.nvfp4_quantize_2d(W.T.copy())
    assert g == gt
    assert np.array_equal(O.nvfp4_unpack(ct), O.nvfp4_unpack(c).T)
    i, j = np.meshgrid(np.arange(48), np.arange(64), indexing="ij")
    assert np.array_equal(sft[j, i // 16], sf[i, j // 16])
    # a row-wise (1 x 16) quantiser does not have this property on the same data
    c1, sf1, _ = O.nvfp4_quantize(W)
    c1t, _, _ = O.nvfp4_quantize(W.T.copy())
    assert not np.array_equal(O.nvfp4_unpack(c1t), O.nvfp4_unpack(c1).T)


def test_nvfp4_2d_equals_1d_when_block_rows_repeat():
    rng = np.random.default_rng(12)
    base = O.round_bf16(rng.standard_normal((3, 80)))
    W = np.repeat(base, 16, axis=0)               # every 16-row block: one row repeated
    c2, s2, g2 = O.nvfp4_quantize_2d(W)
    c1, s1, g1 = O.nvfp4_quantize(W)
    assert g1 == g2 and np.array_equal(c1, c2) and np.array_equal(s1, s2)


@pytest.mark.parametrize("s_g", [1.0, 2.0 ** -4])
def test_nvfp4_2d_round_trip_exact(s_g):
    """Blocks of grid points times a power-of-two block scale, one entry +-6 per
    16 x 16 block: every fp32 step is exact and the round trip is the identity."""
    rng = np.random.default_rng(13)
    rows, cols = 32, 48
    X = np.zeros((rows, cols))
    for rb in range(rows // 16):
        for cb in range(cols // 16):
            sb = 2.0 ** rng.integers(-5, 8)
            q = rng.choice(O.E2M1_MAG, (16, 16)) * rng.choice([-1.0, 1.0], (16, 16))
            q[rng.integers(16), rng.integers(16)] = 6.0
            X[rb * 16:(rb + 1) * 16, cb * 16:(cb + 1) * 16] = q * sb * s_g
    codes, sf, g = O.nvfp4_quantize_2d(X, s_g)
    assert np.array_equal(O.nvfp4_dequantize(codes, sf, g), X)


def test_nvfp4_2d_brute_force_ragged_rows():
    """Rows not a multiple of 16: the last block's scale comes from its rows
    only; every scale and code checked element by element."""
    rng = np.random.default_rng(14)
    W = O.round_bf16(rng.standard_normal((21, 32)) * np.exp(rng.uniform(-2, 2, (21, 2)).repeat(16, axis=1)))
    codes, sf, s_g = O.nvfp4_quantize_2d(W)
    q = O.nvfp4_unpack(codes)
    for rb in range(2):
        r0, r1 = rb * 16, min(21, rb * 16 + 16)
        for cb in range(2):
            blk = W[r0:r1, cb * 16:(cb + 1) * 16]
            amax = np.float32(np.max(np.abs(blk)))
            r_f32 = np.float32(amax / np.float32(np.float32(s_g) * np.float32(6.0)))
            code = torch.tensor([float(r_f32)]).to(torch.float8_e4m3fn).view(torch.uint8).item()
            assert np.all(sf[r0:r1, cb] == code)
            sb = O.e4m3_decode(code)
            sc = np.float32(np.float32(sb) * np.float32(s_g))
            for r in range(r0, r1):
                for i in range(16):
                    v = float(np.float32(np.float32(W[r, cb * 16 + i]) / sc)) if sb != 0 else 0.0
                    assert q[r, cb * 16 + i] == (_brute_e2m1(v) if sb != 0 else 0)
