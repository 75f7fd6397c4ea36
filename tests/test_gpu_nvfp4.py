"""GPU parity of the NVFP4 quantiser (bit-exact codes, scales and global
scale against the oracle) and of the NVFP4 layer forward.

NVFP4 as named on the greeksharifa page, section 2.4 "NVFP4 Training": E2M1
elements, 16-element micro-blocks, E4M3 block scales, an FP32 global scale.
"""
import numpy as np
import pytest
import torch

import lmoe_inputs as LI
from oracle import lmoe_oracle as O

pytestmark = pytest.mark.gpu

L = pytest.importorskip("latentmoe_fwd_b200")
import nvfp4_ties  # noqa: E402
from gpu_util import DevLayer, as_f64, quantize_dev  # noqa: E402


def _bf16_dev(v: np.ndarray):
    bits = LI.bf16_bits(v)
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda(), O.from_bf16_bits(bits)


def _tiled_to_rowmajor(sf_tiled: np.ndarray, rows: int, cols: int) -> np.ndarray:
    """Undo the documented MMA-tiled scale layout."""
    nb = cols // 16
    g64 = (cols + 63) // 64
    out = np.empty((rows, nb), dtype=np.uint8)
    r = np.arange(rows)[:, None]
    j = np.arange(nb)[None, :]
    off = ((r >> 7) * g64 + (j >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (j & 3)
    out[:] = sf_tiled[off]
    return out


@pytest.mark.parametrize("rows,cols,scale", [(1, 16, 1.0), (7, 48, 3.0), (300, 2048, 1.0), (129, 256, 1e-3),
                                            (64, 1024, 50.0)])
def test_quantize_bf16_bit_exact(rows, cols, scale):
    rng = np.random.default_rng(rows * 31 + cols)
    v = rng.standard_normal((rows, cols)) * scale
    v[rng.random((rows, cols)) < 0.001] *= 50.0            # outliers, as in the NVFP4 workload
    x, xv = _bf16_dev(v)
    codes, sf, g = quantize_dev(x, rows, cols)
    rc, rsf, rg = O.nvfp4_quantize(xv)
    assert g.item() == np.float32(rg)
    assert np.array_equal(sf.cpu().numpy(), rsf)
    assert np.array_equal(codes.cpu().numpy(), rc)


def test_quantize_f32_input_and_given_global_scale():
    rng = np.random.default_rng(5)
    v = (rng.standard_normal((40, 160)) * 7).astype(np.float32)
    x = torch.from_numpy(v).cuda()
    gin = torch.tensor([0.0123], dtype=torch.float32, device="cuda")
    codes, sf, g = quantize_dev(x, 40, 160, global_in=gin)
    rc, rsf, rg = O.nvfp4_quantize(v.astype(np.float64), float(np.float32(0.0123)))
    assert g.item() == np.float32(rg)
    assert np.array_equal(sf.cpu().numpy(), rsf)
    assert np.array_equal(codes.cpu().numpy(), rc)


def test_quantize_zero_blocks_and_all_zero_tensor():
    v = np.zeros((3, 64))
    v[1, 20] = -2.5
    x, xv = _bf16_dev(v)
    codes, sf, g = quantize_dev(x, 3, 64)
    rc, rsf, rg = O.nvfp4_quantize(xv)
    assert np.array_equal(codes.cpu().numpy(), rc) and np.array_equal(sf.cpu().numpy(), rsf)
    x0, _ = _bf16_dev(np.zeros((2, 32)))
    c0, s0, g0 = quantize_dev(x0, 2, 32)
    assert g0.item() == 1.0 and not c0.cpu().numpy().any() and not s0.cpu().numpy().any()


@pytest.mark.parametrize("rows,cols", [(128, 64), (300, 2048), (5, 48)])
def test_quantize_mma_tiled_layout(rows, cols):
    rng = np.random.default_rng(rows + cols)
    x, xv = _bf16_dev(rng.standard_normal((rows, cols)))
    codes, sf, g = quantize_dev(x, rows, cols, layout=L.SF_MMA_TILED)
    rc, rsf, rg = O.nvfp4_quantize(xv)
    assert np.array_equal(codes.cpu().numpy(), rc)
    tiled = sf.cpu().numpy()
    assert np.array_equal(_tiled_to_rowmajor(tiled, rows, cols), rsf)
    # every byte outside the real rows/blocks is zero padding
    mask = np.zeros(tiled.size, dtype=bool)
    r = np.arange(rows)[:, None]
    j = np.arange(cols // 16)[None, :]
    g64 = (cols + 63) // 64
    mask[(((r >> 7) * g64 + (j >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (j & 3)).ravel()] = True
    assert not tiled[~mask].any()


def test_hardware_e4m3_conversion_sweep():
    """With s_g = fp32(1/6), s_g * 6 rounds to exactly 1, so each block's scale
    code is the device's E4M3 conversion of the block amax: sweep every E4M3
    value, every midpoint and +-1 fp32 ulp around each, plus random values."""
    mags = O.E4M3_MAG[1:]
    mids = (O.E4M3_MAG[1:] + O.E4M3_MAG[:-1]) / 2
    pts = np.concatenate([mags, mids, [448.0 * 1.01, 460.0, 500.0, 1e4]]).astype(np.float32)
    pts = np.concatenate([pts, np.nextafter(pts, np.float32(np.inf)), np.nextafter(pts, np.float32(0))])
    rng = np.random.default_rng(17)
    pts = np.concatenate([pts, np.exp(rng.uniform(np.log(2e-3), np.log(460), 1 << 16)).astype(np.float32)])
    pts = pts[pts > 0]
    v = np.zeros((pts.size, 16), dtype=np.float32)
    v[:, 0] = pts
    x = torch.from_numpy(v).cuda()
    gin = torch.tensor([1.0 / 6.0], dtype=torch.float32, device="cuda")
    assert np.float32(np.float32(1.0 / 6.0) * np.float32(6.0)) == 1.0
    _, sf, _ = quantize_dev(x, pts.size, 16, global_in=gin)
    assert np.array_equal(sf.cpu().numpy()[:, 0], O.e4m3_encode(pts.astype(np.float64)))


def test_hardware_e2m1_conversion_sweep():
    """Blocks whose amax is 6 get scale E4M3(6) = 6 and s_b * s_g = 1, so every
    other element's code is the device's E2M1 conversion of the element:
    sweep the grid, every midpoint, +-1 fp32 ulp around them, and random values."""
    grid = O.E2M1_MAG
    mids = (grid[1:] + grid[:-1]) / 2
    base = np.concatenate([grid, mids, [6.5, 7.0]]).astype(np.float32)
    base = np.concatenate([base, np.nextafter(base, np.float32(np.inf)), np.nextafter(base, np.float32(0))])
    rng = np.random.default_rng(23)
    vals = np.concatenate([base, -base, rng.uniform(-6, 6, 15 * 4096).astype(np.float32)])
    nblk = (vals.size + 14) // 15
    v = np.zeros((nblk, 16), dtype=np.float32)
    v[:, 0] = 6.0
    flat = np.zeros(nblk * 15, dtype=np.float32)
    flat[:vals.size] = vals
    v[:, 1:] = flat.reshape(nblk, 15)
    v[np.abs(v) > 6] = np.sign(v[np.abs(v) > 6]) * 6.0    # keep each block's amax at 6
    x = torch.from_numpy(v).cuda()
    gin = torch.tensor([1.0 / 6.0], dtype=torch.float32, device="cuda")
    codes, sf, _ = quantize_dev(x, nblk, 16, global_in=gin)
    assert np.all(O.e4m3_decode(sf.cpu().numpy()) == 6.0)
    got = O.nvfp4_unpack(codes.cpu().numpy())
    assert np.array_equal(got, O.e2m1_encode(v.astype(np.float64)))


def prequantize_experts(W, experts, threads=16):
    """Fill the oracle weights view's NVFP4 cache for W1 and W2 of the given
    experts on a thread pool (the quantiser is array code, so threads overlap)."""
    import concurrent.futures as cf
    quant = O.nvfp4_quantize_2d if getattr(W.wl, "w_block2d", False) else O.nvfp4_quantize
    todo = [(k, int(e)) for e in experts for k in ("w1", "w2") if (k, int(e)) not in W._q]

    def one(ke):
        k, e = ke
        return ke, quant(O.to_f64(W.inp[k][e], W.st))

    with cf.ThreadPoolExecutor(threads) as ex:
        for ke, q in ex.map(one, todo):
            W._q[ke] = q


def nvfp4_token_errors(wl, inp, out, gidx, toks, tol):
    """Per-token max|err| beyond half a BF16 step, relative to RMS(oracle out),
    for the given tokens; tokens over `tol` whose latent z has code-changing
    rounding near-ties are re-compared against every alternative rounding."""
    W = O.weights_view(wl, inp, cache=True)
    prequantize_experts(W, np.unique(gidx[toks]))
    ref = O.forward(wl, inp, tokens=toks, idx_override=gidx[toks], weights=W)
    rms = np.sqrt(np.mean(ref["out"] ** 2))

    def excess(got, exact, rounded):
        _, e = np.frexp(np.abs(rounded))
        half = np.ldexp(1.0, np.maximum(e - 1, -126) - 7) / 2
        return np.max(np.maximum(0.0, np.abs(got - exact) - half), axis=-1) / rms

    err = excess(out[toks], ref["out_unrounded"], ref["out"])
    bad = np.where(err > tol)[0]
    n_var = 0
    if bad.size:
        zx, tnorm = nvfp4_ties.z_exact(inp, toks[bad])
        pairs, rows = [], []
        for i, b in enumerate(bad):
            zr, ties = nvfp4_ties.code_changing_ties(zx[i], ref["z_global_scale"], tnorm[i])
            for row in nvfp4_ties.variant_rows(zr, ties):
                pairs.append(b)
                rows.append(row)
        if rows:
            pt = toks[np.array(pairs)]
            alt = O.forward(wl, inp, tokens=pt, idx_override=gidx[pt], z_rows=np.stack(rows), weights=W)
            e_alt = excess(out[pt], alt["out_unrounded"], alt["out"])
            for b, e in zip(pairs, e_alt):
                err[b] = min(err[b], e)
            n_var = len(rows)
        still = [int(b) for b in bad if err[b] > tol]
        if still:
            print(f"{wl.name}: tokens over {tol} after the z-rounding variants: "
                  f"{[(int(toks[b]), round(float(err[b]), 4)) for b in still[:8]]}")
    return err, bad.size, n_var


def _nvfp4_layer(wl, tol=8e-2):
    inp = LI.make_inputs(wl)
    dev = DevLayer(wl, inp)
    out = as_f64(dev.forward())
    gidx, _, _ = dev.route()
    ref = O.forward(wl, inp)
    near = O.near_tie_tokens(ref["logits"], wl.K)
    same = np.all(gidx == ref["idx"], axis=1)
    assert np.all(same | near)
    toks = np.arange(wl.T)
    err, n_tied, n_var = nvfp4_token_errors(wl, inp, out, gidx, toks, tol)
    worst = np.argsort(-err)[:3]
    print(f"{wl.name} T={wl.T}: max|err| beyond BF16 half-step {err.max():.3e} * RMS (median "
          f"{np.median(err):.3e}); {n_tied} tokens re-checked against {n_var} z-rounding variants; "
          f"worst {worst.tolist()} {err[worst].round(4).tolist()}")
    assert err.max() <= tol
    return dev, inp


def test_nvfp4_weights_quantised_bit_exact_per_expert():
    wl = LI.reduced("ultra_nvfp4", T=64, d=256, l=256, N=4, K=2, m=512)
    inp = LI.make_inputs(wl)
    dev = DevLayer(wl, inp)
    w1 = O.from_bf16_bits(inp["w1"])
    codes = dev.t["w1"].cpu().numpy()
    sf = dev.w._keep["w1_sf"].cpu().numpy()
    gs = dev.w._keep["w1_gs"].cpu().numpy()
    for e in range(wl.N):
        rc, rsf, rg = O.nvfp4_quantize(w1[e])
        assert np.array_equal(codes[e], rc)
        assert np.array_equal(_tiled_to_rowmajor(sf[e], wl.m, wl.l), rsf)
        assert gs[e] == np.float32(rg)


@pytest.mark.parametrize("T", [130, 700, 1000, 2100])
def test_nvfp4_forward_reduced(T):
    wl = LI.reduced("ultra_nvfp4", T=T, d=512, l=256, N=16, K=4, m=512)
    _nvfp4_layer(wl)


def test_quantize_codes_at_e2m1_boundaries_with_irregular_scales():
    """Elements at k * sc and a few fp32 ulp around it, for every E2M1 rounding
    boundary k and irregular block scales sc = dec(s_b) * s_g: the device must
    reproduce the codes of RN(x / sc) exactly (it multiplies by RN(1/sc) and
    falls back to the quotient only near a boundary)."""
    rng = np.random.default_rng(29)
    f32 = np.float32
    bounds = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], dtype=np.float32)
    s_g = f32(0.0137)
    t = f32(s_g * f32(6.0))
    blocks = []
    for D in rng.choice(O.E4M3_MAG[8:120], 40):          # normal E4M3 block scales
        D = f32(D)
        amax = f32(D * t)                                   # block max -> scale code D
        sc = f32(f32(O.e4m3_decode(O.e4m3_encode(f32(amax / t)))) * s_g)
        vals = []
        for k in bounds:
            base = f32(k * sc)
            for step in (-3, -2, -1, 0, 1, 2, 3):
                v = base
                for _ in range(abs(step)):
                    v = np.nextafter(v, f32(np.inf) if step > 0 else f32(0))
                vals.append(v)
        vals = np.array(vals, dtype=np.float32)
        for i in range(0, len(vals), 15):
            blk = np.zeros(16, dtype=np.float32)
            blk[0] = amax
            chunk = vals[i:i + 15] * rng.choice([-1, 1], len(vals[i:i + 15])).astype(np.float32)
            blk[1:1 + len(chunk)] = chunk
            blocks.append(blk)
    v = np.stack(blocks)
    x = torch.from_numpy(v).cuda()
    gin = torch.tensor([float(s_g)], dtype=torch.float32, device="cuda")
    codes, sf, _ = quantize_dev(x, v.shape[0], 16, global_in=gin)
    rc, rsf, _ = O.nvfp4_quantize(v.astype(np.float64), float(s_g))
    assert np.array_equal(sf.cpu().numpy(), rsf)
    assert np.array_equal(codes.cpu().numpy(), rc)


# ---- two-dimensional (16 x 16) weight scale blocks ----

@pytest.mark.parametrize("rows,cols", [(48, 64), (21, 96), (300, 2048), (1, 16)])
def test_quantize_2d_bit_exact(rows, cols):
    rng = np.random.default_rng(rows * 17 + cols)
    v = rng.standard_normal((rows, cols)) * np.exp(rng.uniform(-3, 3, (rows, 1)))
    x, xv = _bf16_dev(v)
    codes, sf, g = quantize_dev(x, rows, cols, L.SF_ROWMAJOR | L.SF_BLOCK_16X16)
    rc, rsf, rg = O.nvfp4_quantize_2d(xv)
    assert g.item() == np.float32(rg)
    assert np.array_equal(sf.cpu().numpy(), rsf)
    assert np.array_equal(codes.cpu().numpy(), rc)


def test_quantize_2d_f32_input_given_global_and_tiled_layout():
    rng = np.random.default_rng(21)
    rows, cols = 200, 320                       # ragged last 16-row block and 128-row tile
    v = (rng.standard_normal((rows, cols)) * 3).astype(np.float32)
    x = torch.from_numpy(v).cuda()
    gin = torch.tensor([0.0071], dtype=torch.float32, device="cuda")
    codes, sf, g = quantize_dev(x, rows, cols, L.SF_MMA_TILED | L.SF_BLOCK_16X16, global_in=gin)
    rc, rsf, rg = O.nvfp4_quantize_2d(v.astype(np.float64), float(np.float32(0.0071)))
    assert g.item() == np.float32(rg)
    assert np.array_equal(codes.cpu().numpy(), rc)
    sfn = sf.cpu().numpy()
    assert np.array_equal(_tiled_to_rowmajor(sfn, rows, cols), rsf)
    # padding rows of the last 128-row tile carry zero scales
    pad = np.ones(sfn.shape, dtype=bool)
    r = np.arange(rows)[:, None]
    j = np.arange(cols // 16)[None, :]
    g64 = (cols + 63) // 64
    pad[((r >> 7) * g64 + (j >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (j & 3)] = False
    assert np.all(sfn[pad] == 0)


def test_quantize_2d_transpose_property_on_device():
    rng = np.random.default_rng(22)
    v = rng.standard_normal((64, 96)) * np.exp(rng.uniform(-2, 2, (64, 1)))
    x, xv = _bf16_dev(v)
    xt = x.t().contiguous()
    c, sf, g = quantize_dev(x, 64, 96, L.SF_ROWMAJOR | L.SF_BLOCK_16X16)
    ct, sft, gt = quantize_dev(xt, 96, 64, L.SF_ROWMAJOR | L.SF_BLOCK_16X16)
    assert g.item() == gt.item()
    assert np.array_equal(O.nvfp4_unpack(ct.cpu().numpy()), O.nvfp4_unpack(c.cpu().numpy()).T)
    i, jj = np.meshgrid(np.arange(64), np.arange(96), indexing="ij")
    assert np.array_equal(sft.cpu().numpy()[jj, i // 16], sf.cpu().numpy()[i, jj // 16])


@pytest.mark.parametrize("T", [130, 700])
def test_nvfp4_forward_with_16x16_weight_blocks(T):
    # the block-scaled GEMMs read 2-D-scaled weights unchanged (their scales
    # repeated over each block's 16 rows); parity against the oracle with the
    # same 2-D quantisation of W1 and W2
    wl = LI.reduced("ultra_nvfp4", T=T, d=512, l=256, N=16, K=4, m=512, w_block2d=True)
    _nvfp4_layer(wl)
