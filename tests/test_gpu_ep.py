"""lmoe_ep_reorder on the GPU: the (source, expert) row-block moves of an
expert-parallel plan, both directions, bit-exact against the same moves done
on the host."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

L = pytest.importorskip("latentmoe_fwd_b200")


def test_ep_reorder_both_directions_bit_exact():
    rng = np.random.default_rng(4)
    G, N, l = 3, 10, 96
    counts = rng.integers(0, 40, size=(G, N)).astype(np.int32)
    counts[1, 2] = 0                                    # empty blocks
    plan = L.ep_plan(G, 1, counts)
    n_recv = int(plan["recv_counts"].sum())
    P = int(plan["local_padded_offsets"][-1])
    recv = torch.randn((n_recv, l), device="cuda").to(torch.bfloat16)
    src = torch.from_numpy(plan["block_src"]).cuda()
    dst = torch.from_numpy(plan["block_dst"]).cuda()
    prefix = torch.from_numpy(np.cumsum(plan["block_rows"]).astype(np.int64)).cuda()
    grouped = torch.zeros((P, l), dtype=torch.bfloat16, device="cuda")
    L.ep_reorder(recv, grouped, l * 2, src, dst, prefix, n_recv)
    back = torch.zeros_like(recv)
    L.ep_reorder(grouped, back, l * 2, dst, src, prefix, n_recv)
    torch.cuda.synchronize()
    r, g = recv.cpu(), grouped.cpu()
    ref = torch.zeros_like(g)
    for s, d, c in zip(plan["block_src"], plan["block_dst"], plan["block_rows"]):
        ref[d:d + c] = r[s:s + c]
    assert torch.equal(g, ref)
    assert torch.equal(back.cpu(), r)                   # the way back restores the received order


def _ep_case(G=3, N=12, K=3, l=256, m=256, Ts=(100, 150, 80), seed=7, unused=()):
    """Routing, latent rows and expert weights of a small layer whose tokens
    are split over G emulated ranks (consecutive chunks); experts in `unused`
    receive no token."""
    rng = np.random.default_rng(seed)
    T = sum(Ts)
    p = 1.0 / np.arange(1, N + 1) ** 1.1
    p = p[rng.permutation(N)]
    p[list(unused)] = 0.0
    p = p / p.sum()                                     # skewed expert loads
    idx = np.stack([rng.choice(N, K, replace=False, p=p) for _ in range(T)]).astype(np.int32)
    g = rng.random((T, K)).astype(np.float32) + 0.1
    g = (g / g.sum(axis=1, keepdims=True)).astype(np.float32)
    z = (torch.randn((T, l), device="cuda", generator=torch.Generator("cuda").manual_seed(seed))).to(torch.bfloat16)
    gen = torch.Generator("cuda").manual_seed(seed + 1)
    w1 = (torch.randn((N, m, l), device="cuda", generator=gen) / l ** 0.5).to(torch.bfloat16)
    w2 = (torch.randn((N, l, m), device="cuda", generator=gen) / m ** 0.5).to(torch.bfloat16)
    return dict(G=G, N=N, K=K, l=l, m=m, Ts=list(Ts), T=T, idx=idx, g=g, z=z, w1=w1, w2=w2)


def _one_gpu(c):
    """permute -> expert FFN (gates in GEMM 2) -> combine over all tokens."""
    T, N, K, l, m = c["T"], c["N"], c["K"], c["l"], c["m"]
    cfg = L.config(T=T, d=l, l=l, N=N, K=K, m=m)
    i32 = lambda n: torch.zeros(n, dtype=torch.int32, device="cuda")
    idx = torch.from_numpy(c["idx"]).cuda()
    g = torch.from_numpy(c["g"]).cuda()
    off, ps, inv, poff = i32(N + 1), i32(T * K), i32(T * K), i32(N + 1)
    P = L.padded_rows(cfg)
    zp = torch.zeros((P, l), dtype=torch.bfloat16, device="cuda")
    pg = torch.zeros(P, dtype=torch.float32, device="cuda")
    L.permute(cfg, idx, off, ps, inv, poff, rows=c["z"], row_bytes=l * 2, permuted_rows=zp, topk_w=g, perm_gate=pg,
              ws=L.workspace(cfg, L.OP_PERMUTE))
    y = torch.zeros((P, l), dtype=torch.bfloat16, device="cuda")
    L.expert_ffn(cfg, L.weights(w1=c["w1"], w2=c["w2"]), zp, None, None, off, poff, pg, y,
                 L.workspace(cfg, L.OP_EXPERT_FFN))
    out = torch.empty((T, l), dtype=torch.bfloat16, device="cuda")
    L.combine(cfg, y, idx, inv, off, poff, None, out)
    torch.cuda.synchronize()
    return out


def _expert_parallel(c, corrupt_base=False):
    """The same layer over G emulated ranks on this GPU: every rank permutes
    its own tokens, the counts are exchanged, each rank dispatches its rows
    and gates into the owners' buffers (peer pointers here all point into
    this GPU's memory), each owner runs its experts, each rank combines."""
    G, N, K, l, m, Ts = c["G"], c["N"], c["K"], c["l"], c["m"], c["Ts"]
    i32 = lambda n: torch.zeros(n, dtype=torch.int32, device="cuda")
    starts = np.concatenate([[0], np.cumsum(Ts)])
    ranks = []
    for r in range(G):
        t0, t1 = starts[r], starts[r + 1]
        cfg = L.config(T=Ts[r], d=l, l=l, N=N, K=K, m=m)
        idx = torch.from_numpy(np.ascontiguousarray(c["idx"][t0:t1])).cuda()
        off, ps, inv, poff = i32(N + 1), i32(Ts[r] * K), i32(Ts[r] * K), i32(N + 1)
        L.permute(cfg, idx, off, ps, inv, poff, ws=L.workspace(cfg, L.OP_PERMUTE))
        torch.cuda.synchronize()
        ranks.append(dict(idx=idx, off=off, inv=inv, z=c["z"][t0:t1], g=torch.from_numpy(c["g"][t0:t1].copy()).cuda(),
                          counts=np.diff(off.cpu().numpy())))
    counts = np.stack([rk["counts"] for rk in ranks]).astype(np.int32)   # the count exchange
    plans = [L.ep_plan(G, h, counts) for h in range(G)]
    cap = max(int(p["local_padded_offsets"][-1]) for p in plans)
    recv = [torch.zeros((cap, l), dtype=torch.bfloat16, device="cuda") for _ in range(G)]
    gate = [torch.zeros(cap, dtype=torch.float32, device="cuda") for _ in range(G)]
    ys = [torch.zeros((cap, l), dtype=torch.bfloat16, device="cuda") for _ in range(G)]
    addrs = lambda ts: torch.tensor([t.data_ptr() for t in ts], dtype=torch.int64, device="cuda")
    peer_rows, peer_gates, peer_y = addrs(recv), addrs(gate), addrs(ys)
    err = torch.zeros(64, dtype=torch.int32, device="cuda")
    for r, rk in enumerate(ranks):
        owner, base = L.ep_slot_bases(G, r, counts)
        if corrupt_base and r == 0:
            base = base.copy()
            base[int(rk["idx"][0, 0])] = cap               # rank 0's rows of this expert out of range
        rk["owner"] = torch.from_numpy(owner).cuda()
        rk["base"] = torch.from_numpy(base).cuda()
        L.ep_dispatch(Ts[r], K, N, G, rk["z"], l * 2, rk["idx"], rk["inv"], rk["off"], rk["owner"], rk["base"],
                      peer_rows, cap, rk["g"], peer_gates, err)
    torch.cuda.synchronize()                                # the barrier between the phases
    for h, plan in enumerate(plans):
        f0, nl = plan["first_expert"], plan["local_experts"]
        cfg_h = L.config(T=c["T"], d=l, l=l, N=nl, K=K, m=m)  # T, K bound the owner's padded rows
        off_h = torch.from_numpy(plan["local_offsets"].copy()).cuda()
        poff_h = torch.from_numpy(plan["local_padded_offsets"].copy()).cuda()
        L.expert_ffn(cfg_h, L.weights(w1=c["w1"][f0:f0 + nl], w2=c["w2"][f0:f0 + nl]), recv[h], None, None, off_h,
                     poff_h, gate[h], ys[h], L.workspace(cfg_h, L.OP_EXPERT_FFN))
    torch.cuda.synchronize()
    outs = []
    for r, rk in enumerate(ranks):
        o = torch.empty((Ts[r], l), dtype=torch.bfloat16, device="cuda")
        L.ep_combine(Ts[r], K, N, G, l, peer_y, cap, rk["idx"], rk["inv"], rk["off"], rk["owner"], rk["base"], o, err)
        outs.append(o)
    torch.cuda.synchronize()
    return torch.cat(outs), L.read_device_error(err.view(torch.uint8))


@pytest.mark.parametrize("case", ["three_ranks", "one_rank", "empty_rank_unused_expert"])
def test_ep_dispatch_and_combine_equal_the_one_gpu_layer(case):
    # (tokens x K >= 64 x experts in every case, so the owners' expert GEMMs
    # take the same CTA-pair kernel as the single-GPU reference)
    c = {"three_ranks": lambda: _ep_case(),
         "one_rank": lambda: _ep_case(G=1, Ts=(300,), seed=3),
         "empty_rank_unused_expert": lambda: _ep_case(Ts=(150, 0, 120), seed=5, unused=(4,))}[case]()
    ref = _one_gpu(c)
    got, (st, info) = _expert_parallel(c)
    assert st == L.OK, (st, info)
    # every row and gate lands where the owner's expert GEMMs expect it, and the
    # k-ordered sums read them back: bit for bit the single-GPU result
    assert torch.equal(got, ref)


def test_ep_dispatch_skips_and_reports_rows_out_of_range():
    c = _ep_case(G=2, N=8, K=2, Ts=(160, 200), seed=11)
    ref = _one_gpu(c)
    got, (st, info) = _expert_parallel(c, corrupt_base=True)
    assert st == L.ERR_DEVICE_BOUNDS
    bad = int(c["idx"][0, 0])
    hit = np.zeros(c["T"], dtype=bool)                      # tokens with a slot of the corrupted expert on rank 0
    hit[:c["Ts"][0]] = (c["idx"][:c["Ts"][0]] == bad).any(axis=1)
    assert torch.equal(got[~torch.from_numpy(hit).cuda()], ref[~torch.from_numpy(hit).cuda()])
