"""GPU parity of the router top-K and the expert-grouped permutation.

Routing and permutation are integer results: they must be bit-exact against
the oracle. The GPU router is fed the oracle's logits (rounded to fp32, the
precision the kernel decides in); gates within 1e-6.
"""
import numpy as np
import pytest
import torch

import lmoe_inputs as LI
from oracle import lmoe_oracle as O

pytestmark = pytest.mark.gpu

L = pytest.importorskip("latentmoe_fwd_b200")


def _route_from_logits(logits32, N, K):
    T = logits32.shape[0]
    cfg = L.config(T=T, d=8, l=8, N=N, K=K, m=8)
    idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
    w = torch.empty((T, K), dtype=torch.float32, device="cuda")
    ws = L.workspace(cfg, L.OP_ROUTE)
    lg = torch.from_numpy(np.ascontiguousarray(logits32)).cuda()
    L.route(cfg, None, None, None, lg, idx, w, None, ws)
    st, _ = L.read_device_error(ws)
    assert st == L.OK
    return idx.cpu().numpy(), w.cpu().numpy()


@pytest.mark.parametrize("T,N,K", [(1, 4, 1), (37, 32, 4), (300, 128, 6), (513, 512, 22), (64, 1024, 32),
                                   (5, 33, 32)])
def test_topk_bit_exact_from_oracle_logits(T, N, K):
    rng = np.random.default_rng(T * 7 + N)
    logits = (rng.standard_normal((T, N)) * 2).astype(np.float32)
    idx, w = _route_from_logits(logits, N, K)
    ridx, rw = O.route_topk(logits.astype(np.float64), K)
    assert np.array_equal(idx, ridx)
    assert np.max(np.abs(w - rw)) <= 1e-6


def test_topk_exact_ties_go_to_lower_index():
    rng = np.random.default_rng(3)
    logits = rng.integers(-3, 4, size=(200, 64)).astype(np.float32)   # many exact ties
    idx, w = _route_from_logits(logits, 64, 8)
    ridx, rw = O.route_topk(logits.astype(np.float64), 8)
    assert np.array_equal(idx, ridx)
    assert np.max(np.abs(w - rw)) <= 1e-6


def test_topk_signed_zeros_tie_to_lower_index():
    logits = np.full((3, 40), -1.0, dtype=np.float32)
    logits[0, 5], logits[0, 9] = np.float32(-0.0), np.float32(0.0)    # equal values: expert 5 first
    logits[1, 9], logits[1, 5] = np.float32(-0.0), np.float32(0.0)
    logits[2, 30], logits[2, 2] = np.float32(0.0), np.float32(-0.0)
    idx, w = _route_from_logits(logits, 40, 2)
    assert idx.tolist() == [[5, 9], [5, 9], [2, 30]]
    assert np.allclose(w, 0.5)


@pytest.mark.parametrize("T", [3, 1100])
def test_route_computed_all_logits_equal(T):
    # zero router weights: every logit is exactly 0, so every candidate is in
    # a tie and gets an exact recompute; the lower index wins each tie
    N, K, d = 512, 22, 256
    cfg = L.config(T=T, d=d, l=d, N=N, K=K, m=64)
    x = torch.randn((T, d), device="cuda").to(torch.bfloat16)
    wr = torch.zeros((N, d), device="cuda", dtype=torch.bfloat16)
    idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
    w = torch.empty((T, K), dtype=torch.float32, device="cuda")
    ws = L.workspace(cfg, L.OP_ROUTE)
    L.route(cfg, x, wr, None, None, idx, w, None, ws)
    st, _ = L.read_device_error(ws)
    assert st == L.OK
    assert np.array_equal(idx.cpu().numpy(), np.tile(np.arange(K, dtype=np.int32), (T, 1)))
    assert np.allclose(w.cpu().numpy(), 1.0 / K, rtol=0, atol=1e-7)


@pytest.mark.parametrize("T", [5, 1500])
def test_route_computed_bit_exact_outside_near_ties(T):
    # logits computed on the device (tensor-core GEMM + exact refinement)
    # against the oracle's fp64 decisions; both refinement layouts (one
    # token per block for small T, eight per block above)
    wl = LI.reduced("ultra_zipf", T=T, d=512, l=64, m=64)
    inp = LI.make_inputs(wl)
    cfg = L.config(T=T, d=wl.d, l=wl.l, N=wl.N, K=wl.K, m=wl.m)
    bits = lambda a: torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    x, wr = bits(inp["x"]), bits(inp["w_router"])
    bias = torch.from_numpy(inp["router_bias"]).cuda()
    idx = torch.empty((T, wl.K), dtype=torch.int32, device="cuda")
    w = torch.empty((T, wl.K), dtype=torch.float32, device="cuda")
    ws = L.workspace(cfg, L.OP_ROUTE)
    L.route(cfg, x, wr, bias, None, idx, w, None, ws)
    st, _ = L.read_device_error(ws)
    assert st == L.OK
    logits = O.router_logits(O.from_bf16_bits(inp["x"]), O.from_bf16_bits(inp["w_router"]), inp["router_bias"])
    ridx, rw = O.route_topk(logits, wl.K)
    srt = -np.sort(-logits, axis=1)[:, :wl.K + 1]
    clear = np.min(srt[:, :-1] - srt[:, 1:], axis=1) >= 1e-5       # rows without a near-tie
    assert clear.mean() > 0.9
    got = idx.cpu().numpy()
    assert np.array_equal(got[clear], ridx[clear])
    assert np.max(np.abs(w.cpu().numpy()[clear] - rw[clear])) <= 1e-6


def test_topk_zipf_biased_logits():
    wl = LI.reduced("ultra_zipf", T=257, d=64, l=32, m=32)
    inp = LI.make_inputs(wl)
    x = O.from_bf16_bits(inp["x"])
    logits = O.router_logits(x, O.from_bf16_bits(inp["w_router"]), inp["router_bias"]).astype(np.float32)
    idx, w = _route_from_logits(logits, wl.N, wl.K)
    ridx, rw = O.route_topk(logits.astype(np.float64), wl.K)
    assert np.array_equal(idx, ridx)
    assert np.max(np.abs(w - rw)) <= 1e-6


def _permute(idx_np, N, with_rows=False, row_elems=64):
    T, K = idx_np.shape
    cfg = L.config(T=T, d=row_elems, l=row_elems, N=N, K=K, m=8)
    dev = lambda shape: torch.empty(shape, dtype=torch.int32, device="cuda")
    offsets, poff = dev(N + 1), dev(N + 1)
    perm_src, inv_perm = dev(T * K), dev(T * K)
    idx = torch.from_numpy(np.ascontiguousarray(idx_np, dtype=np.int32)).cuda()
    ws = L.workspace(cfg, L.OP_PERMUTE)
    P = L.padded_rows(cfg)
    rows = prow = None
    w = pg = None
    if with_rows:
        rows = torch.arange(T * row_elems, dtype=torch.float32, device="cuda").view(T, row_elems)
        prow = torch.full((P, row_elems), -1.0, device="cuda")
        w = torch.rand((T, K), device="cuda")
        pg = torch.full((P,), -1.0, device="cuda")
    L.permute(cfg, idx, offsets, perm_src, inv_perm, poff, rows, row_elems * 4 if with_rows else 0, prow,
              topk_w=w, perm_gate=pg, ws=ws)
    st, info = L.read_device_error(ws)
    assert st == L.OK, (st, info)
    out = dict(offsets=offsets.cpu().numpy(), poff=poff.cpu().numpy(), perm_src=perm_src.cpu().numpy(),
               inv_perm=inv_perm.cpu().numpy())
    if with_rows:
        out.update(rows=rows.cpu().numpy(), prow=prow.cpu().numpy(), w=w.cpu().numpy(), pg=pg.cpu().numpy())
    return out


@pytest.mark.parametrize("T,N,K", [(1, 4, 2), (64, 32, 4), (4096, 128, 6), (32, 512, 22), (3000, 512, 22),
                                   (16384, 512, 22)])
def test_permute_bit_exact(T, N, K):
    rng = np.random.default_rng(T + N)
    idx = np.argsort(rng.random((T, N)), axis=1)[:, :K].astype(np.int32)
    g = _permute(idx, N)
    counts, offsets, perm_src, inv_perm = O.permute(idx, N)
    assert np.array_equal(g["offsets"], offsets)
    assert np.array_equal(g["perm_src"], perm_src)
    assert np.array_equal(g["inv_perm"], inv_perm)
    padded = np.zeros(N + 1, dtype=np.int64)
    padded[1:] = np.cumsum((counts + 127) // 128 * 128)
    assert np.array_equal(g["poff"], padded)


def test_permute_skewed_and_empty_experts():
    rng = np.random.default_rng(9)
    T, N, K = 5000, 64, 3
    # Zipf-like: most slots on a few experts, many experts empty
    p = 1.0 / np.arange(1, N + 1) ** 2.0
    p /= p.sum()
    idx = np.stack([rng.choice(N, K, replace=False, p=p) for _ in range(T)]).astype(np.int32)
    g = _permute(idx, N)
    _, offsets, perm_src, inv_perm = O.permute(idx, N)
    assert np.array_equal(g["offsets"], offsets)
    assert np.array_equal(g["perm_src"], perm_src)
    assert np.array_equal(g["inv_perm"], inv_perm)


def test_permute_gathers_rows_and_gates_to_padded_rows():
    rng = np.random.default_rng(10)
    T, N, K = 300, 16, 4
    idx = np.argsort(rng.random((T, N)), axis=1)[:, :K].astype(np.int32)
    g = _permute(idx, N, with_rows=True)
    _, offsets, perm_src, _ = O.permute(idx, N)
    flat = idx.reshape(-1)
    for r in range(T * K):
        f = perm_src[r]
        e = flat[f]
        p = r - offsets[e] + g["poff"][e]
        assert np.array_equal(g["prow"][p], g["rows"][f // K])
        assert g["pg"][p] == g["w"].reshape(-1)[f]


def test_permute_out_of_range_expert_reports_bounds_error():
    T, N, K = 10, 8, 2
    idx = np.zeros((T, K), dtype=np.int32)
    idx[:, 1] = 1
    idx[3, 0] = 9        # out of range: the host cannot see it, the device reports it
    cfg = L.config(T=T, d=8, l=8, N=N, K=K, m=8)
    dev = lambda n: torch.zeros(n, dtype=torch.int32, device="cuda")
    ws = L.workspace(cfg, L.OP_PERMUTE)
    L.permute(cfg, torch.from_numpy(idx).cuda(), dev(N + 1), dev(T * K), dev(T * K), dev(N + 1), ws=ws)
    st, info = L.read_device_error(ws)
    assert st == L.ERR_DEVICE_BOUNDS
    assert info == 3 * K + 0
    st2, _ = L.read_device_error(ws)
    assert st2 == L.OK          # reading clears the word


def test_out_of_range_expert_is_left_out_of_gather_and_combine():
    """A slot whose expert index is >= N is reported, left out of the sorted
    positions (offsets[N] counts only in-range slots), not gathered, and
    contributes nothing to the combine. Buffers start zeroed, so every index
    the kernels could take stays inside them."""
    T, N, K, l = 10, 8, 2, 64
    idx = np.zeros((T, K), dtype=np.int32)
    idx[:, 1] = 1
    idx[3, 0] = 9
    idx[6, 1] = 8        # == N: out of range as well
    bad = {(3, 0), (6, 1)}
    rng = np.random.default_rng(21)
    rows32 = rng.standard_normal((T, l)).astype(np.float32)
    # powers of two: every gate * row product is exact, so fused and separate
    # multiply-adds round alike and the comparison can be bit-exact
    w = rng.choice([0.25, 0.5, 1.0, 2.0], size=(T, K)).astype(np.float32)
    cfg = L.config(T=T, d=l, l=l, N=N, K=K, m=64)
    P = L.padded_rows(cfg)
    z32 = lambda n: torch.zeros(n, dtype=torch.int32, device="cuda")
    rows = torch.from_numpy(rows32).cuda().to(torch.bfloat16)
    prow = torch.zeros((P, l), dtype=torch.bfloat16, device="cuda")
    pgate = torch.zeros(P, dtype=torch.float32, device="cuda")
    offsets, perm_src, inv_perm, poff = z32(N + 1), z32(T * K), z32(T * K), z32(N + 1)
    idx_d = torch.from_numpy(idx).cuda()
    w_d = torch.from_numpy(w).cuda()
    ws = L.workspace(cfg, L.OP_PERMUTE)
    L.permute(cfg, idx_d, offsets, perm_src, inv_perm, poff, rows, l * 2, prow, None, None, w_d, pgate, ws=ws)
    st, info = L.read_device_error(ws)
    assert st == L.ERR_DEVICE_BOUNDS and info in (3 * K + 0, 6 * K + 1)
    off, pf = offsets.cpu().numpy(), poff.cpu().numpy()
    assert off[N] == T * K - len(bad)
    assert off[1] - off[0] == T - 1 and off[2] - off[1] == T - 1 and off[N] == off[2]
    # exactly the in-range slots are gathered, with their gates; padding stays zero
    expect = torch.zeros((P, l), dtype=torch.bfloat16)
    gexp = torch.zeros(P, dtype=torch.float32)
    ip = inv_perm.cpu().numpy()
    for t in range(T):
        for k in range(K):
            if (t, k) in bad:
                continue
            e = idx[t, k]
            p = ip[t * K + k] - off[e] + pf[e]
            expect[p] = rows[t].cpu()
            gexp[p] = float(w[t, k])
    assert torch.equal(prow.cpu(), expect)
    assert torch.equal(pgate.cpu(), gexp)
    # combine over the gathered rows: c_t = sum over in-range k, fp32 in k order
    c = torch.zeros((T, l), dtype=torch.bfloat16, device="cuda")
    L.combine(cfg, prow, idx_d, inv_perm, offsets, poff, w_d, c)
    torch.cuda.synchronize()
    rb = rows.float().cpu().numpy()
    acc = np.zeros((T, l), dtype=np.float32)
    for t in range(T):
        for k in range(K):
            if (t, k) not in bad:
                acc[t] += np.float32(w[t, k]) * rb[t]
    assert torch.equal(c.cpu(), torch.from_numpy(acc).to(torch.bfloat16))
