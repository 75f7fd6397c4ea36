"""Parity at the workloads' full sizes, in the launch configuration the
benchmark times (lmoe_forward on the whole batch).

* routing over every token: bit-exact against the oracle's selection from its
  own fp64 logits, except documented near-ties (gap < 1e-5);
* the permutation of the GPU's routing: bit-exact over every slot;
* layer outputs: a stratified sample of at least 128 tokens the oracle
  computes one by one -- tokens in the first, a middle and the ragged last
  256-row tile of the heaviest experts, tokens of experts that hold only one
  or two rows, and seeded random tokens -- with two bars: the error beyond
  half a BF16 step of the exact output (2e-2 * RMS BF16, 8e-2 * RMS NVFP4) and
  the raw error against the oracle's BF16-rounded output, element by element,
  within that bar plus one BF16 step of the element;
* expert FFN outputs (lmoe_expert_ffn at full size on the oracle's routing):
  rows from every token tile of every expert, its first, middle and last row,
  so every tile the grouped GEMMs run -- ragged last tiles and one-row
  experts included -- is compared with the oracle.
"""
import functools

import numpy as np
import pytest
import torch

import lmoe_inputs as LI
from oracle import lmoe_oracle as O

pytestmark = pytest.mark.gpu

L = pytest.importorskip("latentmoe_fwd_b200")
from gpu_util import DevLayer, as_f64, bf16_parity, bf16_raw_within, to_dev  # noqa: E402

MIN_SAMPLE = 128
TILE = 256          # tokens per grouped-GEMM tile (CTA pairs); other tile widths divide it


@functools.lru_cache(maxsize=1)
def _oracle_routing(name):
    """Inputs, fp64 logits, the oracle's top-K and gates of a full workload."""
    wl = LI.WORKLOADS[name]
    inp = LI.make_inputs(wl)
    x = O.from_bf16_bits(inp["x"])
    logits = O.router_logits(x, O.from_bf16_bits(inp["w_router"]), inp["router_bias"])
    ridx, rgates = O.route_topk(logits, wl.K)
    return wl, inp, logits, ridx, rgates


def stratified_tokens(idx, N, K, rng, total=MIN_SAMPLE, heavy=8, light=8):
    """Tokens that reach every kind of grouped-GEMM tile, from a routing idx [T, K].

    For the `heavy` experts with the most rows: the tokens at sorted positions
    0 (first tile), the middle of the expert, the first row of its last
    256-row tile and its last row (the ragged tail). For up to `light` experts
    with one or two rows: all their tokens. Then seeded random tokens up to
    `total`. Returns (sorted token array, counts of each stratum)."""
    T = idx.shape[0]
    flat = idx.reshape(-1)
    counts = np.bincount(flat, minlength=N)
    order = np.argsort(flat, kind="stable")          # slots sorted by (expert, slot)
    starts = np.concatenate([[0], np.cumsum(counts)])
    toks, strata = set(), {"heavy": 0, "light": 0, "random": 0}
    for e in np.argsort(-counts, kind="stable")[:heavy]:
        n = int(counts[e])
        if n == 0:
            continue
        last_tile = ((n - 1) // TILE) * TILE
        for pos in {0, n // 2, last_tile, n - 1}:
            toks.add(int(order[starts[e] + pos]) // K)
        strata["heavy"] += 1
    small = [e for e in range(N) if 1 <= counts[e] <= 2][:light]
    for e in small:
        for pos in range(int(counts[e])):
            toks.add(int(order[starts[e] + pos]) // K)
        strata["light"] += 1
    while len(toks) < min(total, T):
        t = int(rng.integers(T))
        if t not in toks:
            toks.add(t)
            strata["random"] += 1
    return np.array(sorted(toks)), strata


@pytest.mark.parametrize("name", ["std_moe_bf16", "ultra_decode", "ultra_zipf"])
def test_full_size_bf16(name):
    wl, inp, logits, ridx, rgates = _oracle_routing(name)
    dev = DevLayer(wl, inp)
    out = as_f64(dev.forward())
    gidx, gw, glogits = dev.route()

    # routing over every token
    near = O.near_tie_tokens(logits, wl.K)
    same = np.all(gidx == ridx, axis=1)
    dl = np.abs(glogits.astype(np.float64) - logits)
    srt = -np.sort(-logits, axis=1)
    gaps = srt[:, :wl.K] - srt[:, 1:wl.K + 1]
    bad = np.where(~same)[0]
    print(f"{name}: logit error max {dl.max():.3e} mean {dl.mean():.3e}; misrouted {bad.size}; "
          f"their min adjacent gap {[float(gaps[t].min()) for t in bad[:16]]}")
    # the router's exact-refinement window assumes the tensor-core logit error
    # stays below tau = 2^-12 * RMS(bias-free logits) + 2^-22 * max|logit|
    nb = glogits.astype(np.float64) - (inp["router_bias"][None, :] if inp["router_bias"] is not None else 0.0)
    tau = np.sqrt(np.mean(nb ** 2, axis=1)) * 2.0 ** -12 + np.max(np.abs(glogits), axis=1) * 2.0 ** -22
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

    # stratified sample of outputs
    toks, strata = stratified_tokens(gidx, N, K, np.random.default_rng(123))
    ref = O.forward(wl, inp, tokens=toks, idx_override=gidx[toks])
    excess, raw = bf16_parity(out[toks], ref["out_unrounded"], ref["out"])
    raw_ok, raw_worst = bf16_raw_within(out[toks], ref["out"], 2e-2)
    print(f"{name}: {len(toks)} tokens {strata}: excess {excess:.3e} * RMS, raw {raw:.3e} * RMS "
          f"(raw / (2e-2 RMS + 1 ulp) max {raw_worst:.3f})")
    assert excess <= 2e-2
    assert raw_ok


def _expert_rows(counts, tile=TILE):
    """Sorted positions to check per expert: first, middle and last row of every token tile."""
    pos = []
    for e, n in enumerate(counts):
        n = int(n)
        for t0 in range(0, n, tile):
            t1 = min(n, t0 + tile)
            for p in sorted({t0, (t0 + t1) // 2, t1 - 1}):
                pos.append((e, p))
    return pos


@pytest.mark.parametrize("name", ["std_moe_bf16", "ultra_zipf"])
def test_full_size_expert_ffn_every_tile(name):
    """lmoe_expert_ffn at full size on the oracle's routing and seeded latent
    rows z ~ N(0, 1) (BF16): rows of every token tile of every expert against
    y = RN(g * (RN(relu(z W1_e^T)^2) W2_e^T)) computed by the oracle's pieces."""
    wl, inp, _, ridx, rgates = _oracle_routing(name)
    T, K, N, l, m = wl.T, wl.K, wl.N, wl.l, wl.m
    rng = np.random.default_rng(777)
    z_bits = LI.bf16_bits(rng.standard_normal((T, l)))
    z = O.from_bf16_bits(z_bits)
    dev = DevLayer(wl, inp)
    cfg = dev.cfg
    P = L.padded_rows(cfg)
    i32 = lambda n: torch.empty(n, dtype=torch.int32, device="cuda")
    offsets, poff, perm_src, inv_perm = i32(N + 1), i32(N + 1), i32(T * K), i32(T * K)
    zp = torch.zeros((P, l), dtype=torch.bfloat16, device="cuda")
    pg = torch.zeros(P, dtype=torch.float32, device="cuda")
    ws = L.workspace(cfg, L.OP_PERMUTE)
    L.permute(cfg, torch.from_numpy(ridx.astype(np.int32)).cuda(), offsets, perm_src, inv_perm, poff,
              to_dev(z_bits, "bf16"), l * 2, zp, topk_w=torch.from_numpy(rgates.astype(np.float32)).cuda(),
              perm_gate=pg, ws=ws)
    assert L.read_device_error(ws)[0] == L.OK
    y = torch.empty((P, l), dtype=torch.bfloat16, device="cuda")
    ws2 = L.workspace(cfg, L.OP_EXPERT_FFN)
    L.expert_ffn(cfg, dev.w, zp, None, None, offsets, poff, pg, y, ws2)
    assert L.read_device_error(ws2)[0] == L.OK
    poff_h = poff.cpu().numpy()

    counts, r_off, r_src, _ = O.permute(ridx, N)
    pos = _expert_rows(counts)
    W = O.weights_view(wl, inp)
    gates32 = rgates.astype(np.float32).astype(np.float64)   # the gate the GPU multiplies by (fp32)
    got_rows, ref_rows, ref_exact = [], [], []
    by_e = {}
    for e, p in pos:
        by_e.setdefault(e, []).append(p)
    prow_all = []
    for e, ps in by_e.items():
        ps = np.array(ps)
        slots = r_src[r_off[e] + ps]
        t, k = slots // K, slots % K
        h = z[t] @ W.expert("w1", e).T
        a = O.rho(O.sq_relu(h), "bf16")
        yx = gates32[t, k][:, None] * (a @ W.expert("w2", e).T)
        ref_exact.append(yx)
        ref_rows.append(O.rho(yx, "bf16"))
        prow_all.append(poff_h[e] + ps)
    prow = torch.from_numpy(np.concatenate(prow_all)).cuda()
    got = as_f64(y[prow])
    ref_r, ref_x = np.concatenate(ref_rows), np.concatenate(ref_exact)
    excess, raw = bf16_parity(got, ref_x, ref_r)
    raw_ok, raw_worst = bf16_raw_within(got, ref_r, 2e-2)
    n_tiles = sum(-(-int(c) // TILE) for c in counts)
    print(f"{name}: {len(pos)} rows from {n_tiles} token tiles of {int(np.count_nonzero(counts))} experts: "
          f"excess {excess:.3e} * RMS, raw {raw:.3e} * RMS (raw / bar max {raw_worst:.3f})")
    assert excess <= 2e-2
    assert raw_ok


def test_full_size_nvfp4_expert_ffn_every_tile():
    """lmoe_expert_ffn on the NVFP4 path at full size (ultra_nvfp4): the
    oracle's routing and its BF16 z quantised on the GPU (the quantiser is
    bit-exact, so both sides start from the same codes), rows of every
    128-row tile of every expert against the oracle's expert FFN with its
    NVFP4 rounding points (z and a fake-quantised, 16-element blocks)."""
    from test_gpu_nvfp4 import prequantize_experts
    from gpu_util import quantize_dev
    name = "ultra_nvfp4"
    wl, inp, _, ridx, rgates = _oracle_routing(name)
    T, K, N, l, m = wl.T, wl.K, wl.N, wl.l, wl.m
    x = O.from_bf16_bits(inp["x"])
    z = O.round_bf16(x @ O.from_bf16_bits(inp["w_down"]).T)          # the oracle's stored z
    dev = DevLayer(wl, inp)
    cfg = dev.cfg
    P = L.padded_rows(cfg)
    zq, zsf, zgs = quantize_dev(to_dev(LI.bf16_bits(z), "bf16"), T, l)
    i32 = lambda n: torch.empty(n, dtype=torch.int32, device="cuda")
    offsets, poff, perm_src, inv_perm = i32(N + 1), i32(N + 1), i32(T * K), i32(T * K)
    zp = torch.zeros((P, l // 2), dtype=torch.uint8, device="cuda")
    zpsf = torch.zeros((P * l // 16,), dtype=torch.uint8, device="cuda")
    pg = torch.zeros(P, dtype=torch.float32, device="cuda")
    ws = L.workspace(cfg, L.OP_PERMUTE)
    L.permute(cfg, torch.from_numpy(ridx.astype(np.int32)).cuda(), offsets, perm_src, inv_perm, poff, zq, l // 2,
              zp, rows_sf=zsf, permuted_sf=zpsf, topk_w=torch.from_numpy(rgates.astype(np.float32)).cuda(),
              perm_gate=pg, ws=ws)
    assert L.read_device_error(ws)[0] == L.OK
    y = torch.empty((P, l), dtype=torch.bfloat16, device="cuda")
    ws2 = L.workspace(cfg, L.OP_EXPERT_FFN)
    L.expert_ffn(cfg, dev.w, zp, zpsf, zgs, offsets, poff, pg, y, ws2)
    assert L.read_device_error(ws2)[0] == L.OK
    poff_h = poff.cpu().numpy()

    counts, r_off, r_src, _ = O.permute(ridx, N)
    pos = _expert_rows(counts, tile=128)
    W = O.weights_view(wl, inp, cache=True)
    prequantize_experts(W, np.nonzero(counts)[0])
    s_z = float(zgs.item())
    assert s_z == np.float32(O.nvfp4_global_scale(z))
    a_gs = inp["a_global_scale"]
    g32 = rgates.astype(np.float32).astype(np.float64)
    by_e = {}
    for e, p in pos:
        by_e.setdefault(e, []).append(p)
    got_rows, ref_rows, ref_exact = [], [], []
    for e, ps in by_e.items():
        ps = np.array(ps)
        slots = r_src[r_off[e] + ps]
        t, k = slots // K, slots % K
        zq_rows = O.nvfp4_fake_quant(z[t], s_z)[0]
        aq = O.nvfp4_fake_quant(O.sq_relu(zq_rows @ W.expert("w1", e).T), a_gs)[0]
        yx = g32[t, k][:, None] * (aq @ W.expert("w2", e).T)
        ref_exact.append(yx)
        ref_rows.append(O.round_bf16(yx))
        got_rows.append(poff_h[e] + ps)
    got = as_f64(y[torch.from_numpy(np.concatenate(got_rows)).cuda()])
    excess, raw = bf16_parity(got, np.concatenate(ref_exact), np.concatenate(ref_rows))
    print(f"{name}: {len(pos)} expert-FFN rows from every 128-row tile: excess {excess:.3e} * RMS, "
          f"raw {raw:.3e} * RMS")
    assert excess <= 8e-2


@pytest.mark.parametrize("name", ["ultra_nvfp4", "ultra_decode_nvfp4", "ultra_nvfp4_fp8shared"])
def test_full_size_nvfp4(name):
    """NVFP4 workloads at full size (the T=8192 layer, the same layer in
    decode, and the T=8192 layer with FP8 shared experts): weights quantised on the GPU (bit-exact per expert against the
    oracle for a sample of experts), routing checked over every token, outputs
    of a stratified token sample within 8e-2 * RMS beyond half a BF16 step,
    allowing the documented z-rounding near-ties."""
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
    # NVFP4 tiles hold 128 rows; the 256-row strata still reach first, middle and last tiles
    toks, strata = stratified_tokens(gidx, wl.N, wl.K, np.random.default_rng(321), total=64)
    err, n_tied, n_var = nvfp4_token_errors(wl, inp, out, gidx, toks, 8e-2)
    print(f"{name}: {len(toks)} tokens {strata}: max|err| beyond BF16 half-step {err.max():.3e} * RMS; "
          f"{n_tied} re-checked against {n_var} variants")
    assert err.max() <= 8e-2
