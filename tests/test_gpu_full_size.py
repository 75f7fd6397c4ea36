"""Parity at the workloads' full sizes, in the launch configuration the
benchmark times (lmoe_forward on the whole batch).

* routing over every token: bit-exact against the oracle's selection from its
  own fp64 logits, except documented near-ties (gap < 1e-5);
* the permutation of the GPU's routing: bit-exact over every slot;
* outputs: a seeded sample of tokens the oracle computes one by one, with the
  same error measure as the reduced-size tests (BF16: max|err| beyond half a
  BF16 step <= 2e-2 * RMS).
"""
import numpy as np
import pytest
import torch

import lmoe_inputs as LI
from oracle import lmoe_oracle as O

pytestmark = pytest.mark.gpu

L = pytest.importorskip("latentmoe_fwd_b200")
from gpu_util import DevLayer, as_f64, bf16_parity  # noqa: E402

SAMPLE = 24


@pytest.mark.parametrize("name", ["std_moe_bf16", "ultra_decode", "ultra_zipf"])
def test_full_size_bf16(name):
    wl = LI.WORKLOADS[name]
    inp = LI.make_inputs(wl)
    dev = DevLayer(wl, inp)
    out = as_f64(dev.forward())
    gidx, gw, glogits = dev.route()

    # routing over every token
    x = O.from_bf16_bits(inp["x"])
    logits = O.router_logits(x, O.from_bf16_bits(inp["w_router"]), inp["router_bias"])
    ridx, rgates = O.route_topk(logits, wl.K)
    near = O.near_tie_tokens(logits, wl.K)
    same = np.all(gidx == ridx, axis=1)
    dl = np.abs(glogits.astype(np.float64) - logits)
    srt = -np.sort(-logits, axis=1)
    gaps = srt[:, :wl.K] - srt[:, 1:wl.K + 1]
    bad = np.where(~same)[0]
    print(f"{name}: logit error max {dl.max():.3e} mean {dl.mean():.3e}; misrouted {bad.size}; "
          f"their min adjacent gap {[float(gaps[t].min()) for t in bad[:16]]}")
    # the router's exact-refinement window assumes the tensor-core logit error
    # stays below tau = 2^-10 * RMS(bias-free logits) + 2^-20 * max|logit|
    nb = glogits.astype(np.float64) - (inp["router_bias"][None, :] if inp["router_bias"] is not None else 0.0)
    tau = np.sqrt(np.mean(nb ** 2, axis=1)) * 2.0 ** -10 + np.max(np.abs(glogits), axis=1) * 2.0 ** -20
    ratio = float(np.max(dl / tau[:, None]))
    print(f"{name}: max logit error / tau = {ratio:.3f}")
    assert ratio < 0.5
    assert np.all(same | near), f"{np.sum(~(same | near))} tokens routed differently without a near-tie"
    ok = same
    assert np.max(np.abs(gw[ok] - rgates[ok])) <= 1e-5
    print(f"{name}: {np.sum(near)} near-tie tokens, {np.sum(~same)} routed differently")

    # permutation of the GPU's routing, every slot
    T, K, N = wl.T, wl.K, wl.N
    cfg = dev.cfg
    i32 = lambda n: torch.empty(n, dtype=torch.int32, device="cuda")
    offsets, poff, perm_src, inv_perm = i32(N + 1), i32(N + 1), i32(T * K), i32(T * K)
    ws = L.workspace(cfg, L.OP_PERMUTE)
    L.permute(cfg, torch.from_numpy(gidx).cuda(), offsets, perm_src, inv_perm, poff, ws=ws)
    assert L.read_device_error(ws)[0] == L.OK
    _, r_off, r_src, r_inv = O.permute(gidx, N)
    assert np.array_equal(offsets.cpu().numpy(), r_off)
    assert np.array_equal(perm_src.cpu().numpy(), r_src)
    assert np.array_equal(inv_perm.cpu().numpy(), r_inv)

    # sampled outputs
    rng = np.random.default_rng(123)
    toks = np.sort(rng.choice(T, size=min(SAMPLE, T), replace=False))
    ref = O.forward(wl, inp, tokens=toks, idx_override=gidx[toks])
    excess, raw = bf16_parity(out[toks], ref["out_unrounded"], ref["out"])
    print(f"{name}: sampled {len(toks)} tokens: excess {excess:.3e} * RMS, raw {raw:.3e} * RMS")
    assert excess <= 2e-2


@pytest.mark.parametrize("name", ["ultra_nvfp4", "ultra_decode_nvfp4"])
def test_full_size_nvfp4(name):
    """NVFP4 workloads at full size (the T=8192 layer and the same layer in
    decode): weights quantised on the GPU (bit-exact per expert against the
    oracle for a sample of experts), routing checked over every token, outputs
    of sampled tokens within 8e-2 * RMS beyond half a BF16 step, allowing the
    documented z-rounding near-ties."""
    from test_gpu_nvfp4 import _tiled_to_rowmajor, nvfp4_token_errors
    wl = LI.WORKLOADS[name]
    inp = LI.make_inputs(wl)
    dev = DevLayer(wl, inp)
    for e in (0, 257, 511):
        rc, rsf, rg = O.nvfp4_quantize(O.from_bf16_bits(inp["w1"][e]))
        assert np.array_equal(dev.t["w1"][e].cpu().numpy(), rc)
        assert np.array_equal(_tiled_to_rowmajor(dev.w._keep["w1_sf"][e].cpu().numpy(), wl.m, wl.l), rsf)
        assert dev.w._keep["w1_gs"][e].item() == np.float32(rg)
    out = as_f64(dev.forward())
    gidx, _, glogits = dev.route()
    x = O.from_bf16_bits(inp["x"])
    logits = O.router_logits(x, O.from_bf16_bits(inp["w_router"]), None)
    ridx, _ = O.route_topk(logits, wl.K)
    near = O.near_tie_tokens(logits, wl.K)
    same = np.all(gidx == ridx, axis=1)
    print(f"{name}: {np.sum(near)} near-tie tokens, {np.sum(~same)} routed differently")
    assert np.all(same | near)
    rng = np.random.default_rng(321)
    toks = np.sort(rng.choice(wl.T, size=min(12, wl.T), replace=False))
    err, n_tied, n_var = nvfp4_token_errors(wl, inp, out, gidx, toks, 8e-2)
    print(f"{name}: sampled {len(toks)} tokens: max|err| beyond BF16 half-step {err.max():.3e} * RMS; "
          f"{n_tied} re-checked against {n_var} variants")
    assert err.max() <= 8e-2
