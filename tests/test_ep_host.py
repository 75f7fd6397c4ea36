"""Expert parallelism in the latent dimension, host side, on CPU: world-size-2
`gloo` ranks each route and permute their own tokens, exchange per-expert
counts, plan the dispatch with lmoe_ep_plan (the library's host code), send
their l-dim rows to the experts' owners with all_to_all_single, run the owned
experts on the expert-grouped rows, send the outputs back and combine. The
sharded layer must equal the oracle's unsharded forward token for token
(fp64, no rounding points), which checks ownership, the count exchange, the
send/receive offsets and both reorders; the same rank processes check the
peer-memory data plane's addressing (lmoe_ep_slot_bases) against it."""
import os
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _reorder(rows, plan, back: bool, n_out: int):
    """Move (source, expert) blocks: received (source-major) -> expert-grouped, or back."""
    out = np.zeros((n_out, rows.shape[1]))
    for s, d, c in zip(plan["block_src"], plan["block_dst"], plan["block_rows"]):
        if back:
            s, d = d, s
        out[d:d + c] = rows[s:s + c]
    return out


def _rank_main(rank, world, port, T_each, result):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import latentmoe_fwd_b200 as L
    import lmoe_inputs as LI
    from oracle import lmoe_oracle as O
    wl = LI.reduced("ultra_decode", T=T_each * world, d=64, l=32, N=7, K=3, m=48)
    inp = LI.make_inputs(wl)                        # same weights on every rank; each takes its tokens
    tok = np.arange(rank * T_each, (rank + 1) * T_each)
    x = O.from_bf16_bits(inp["x"])[tok]
    wr, wd, wu = (O.from_bf16_bits(inp[k]) for k in ("w_router", "w_down", "w_up"))
    w1, w2 = O.from_bf16_bits(inp["w1"]), O.from_bf16_bits(inp["w2"])
    N, K, l = wl.N, wl.K, wl.l
    idx, gates = O.route_topk(O.router_logits(x, wr), K)
    counts, offsets, perm_src, inv_perm = O.permute(idx, N)
    z = x @ wd.T
    zs = z[perm_src // K]                           # this rank's rows in sorted (expert-major) order

    # count exchange: every rank learns the [G][N] count matrix
    parts = [torch.zeros(N, dtype=torch.int32) for _ in range(world)]
    dist.all_gather(parts, torch.from_numpy(counts.astype(np.int32)))
    plan = L.ep_plan(world, rank, torch.stack(parts).numpy())
    assert np.array_equal(plan["send_offsets"][1:], np.cumsum(plan["send_counts"])[:-1])

    # dispatch: l-dim rows to the owners of their experts
    recv = torch.zeros((int(plan["recv_counts"].sum()), l), dtype=torch.float64)
    dist.all_to_all_single(recv, torch.from_numpy(zs), output_split_sizes=plan["recv_counts"].tolist(),
                           input_split_sizes=plan["send_counts"].tolist())
    P = int(plan["local_padded_offsets"][-1])
    grouped = _reorder(recv.numpy(), plan, back=False, n_out=P)
    # the owned experts on their grouped rows (ungated; the source applies its gates)
    y = np.zeros_like(grouped)
    f0 = plan["first_expert"]
    for el in range(plan["local_experts"]):
        n = plan["local_offsets"][el + 1] - plan["local_offsets"][el]
        p0 = plan["local_padded_offsets"][el]
        rows = grouped[p0:p0 + n]
        y[p0:p0 + n] = O.sq_relu(rows @ w1[f0 + el].T) @ w2[f0 + el].T
    # combine: outputs back to their sources, in the sources' sorted order
    back = torch.from_numpy(_reorder(y, plan, back=True, n_out=recv.shape[0]))
    ys = torch.zeros((zs.shape[0], l), dtype=torch.float64)
    dist.all_to_all_single(ys, back, output_split_sizes=plan["send_counts"].tolist(),
                           input_split_sizes=plan["recv_counts"].tolist())
    y_slot = np.zeros((T_each * K, l))
    y_slot[perm_src] = ys.numpy()
    c = np.einsum("tk,tkl->tl", gates, y_slot.reshape(T_each, K, l))

    # the peer-memory data plane's addressing (lmoe_ep_slot_bases, as
    # lmoe_ep_dispatch / lmoe_ep_combine apply it): slot f of expert e goes to
    # rank owner[e], row base[e] + inv_perm[f] - offsets[e]. The stores are
    # emulated by gathering (rank, row, data) at every rank; each owner's
    # buffer must equal the all-to-all + reorder result, and reading the
    # owners' outputs back at the same rows must give this rank's y rows.
    owner, base = L.ep_slot_bases(world, rank, torch.stack(parts).numpy())
    e_slot = idx.reshape(-1)
    dst_rank = owner[e_slot]
    dst_row = base[e_slot] + inv_perm - offsets[e_slot]
    stores = [None] * world
    dist.all_gather_object(stores, (dst_rank, dst_row, z[np.arange(T_each * K) // K]))
    mine = np.zeros((P, l))
    for dr, rr, data in stores:
        sel = dr == rank
        mine[rr[sel]] = data[sel]
    real = np.concatenate([np.arange(plan["local_padded_offsets"][el],
                                     plan["local_padded_offsets"][el] + plan["local_offsets"][el + 1]
                                     - plan["local_offsets"][el]) for el in range(plan["local_experts"])])
    assert np.array_equal(mine[real], grouped[real])
    ys_all = [None] * world
    dist.all_gather_object(ys_all, y)
    y_read = np.stack([ys_all[h][r] for h, r in zip(dst_rank, dst_row)])
    assert np.array_equal(y_read, y_slot)
    out = c @ wu.T
    ref = O.forward(wl, inp, tokens=tok, precision="f64")["out"]
    result[rank] = float(np.max(np.abs(out - ref)) / np.sqrt(np.mean(ref ** 2)))
    dist.barrier()
    dist.destroy_process_group()


def test_expert_parallel_layer_equals_the_unsharded_layer():
    world, T_each = 2, 40
    port = 29900 + os.getpid() % 90
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    result = mgr.dict()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, T_each, result)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    assert set(result.keys()) == {0, 1}
    assert max(result.values()) < 1e-12, dict(result)


def test_ep_plan_layout_on_a_hand_example():
    sys.path.insert(0, ROOT)
    import latentmoe_fwd_b200 as L
    # 2 ranks, 5 experts: rank 0 owns experts 0-2, rank 1 owns 3-4
    counts = np.array([[2, 0, 1, 3, 4],
                       [1, 5, 0, 0, 2]], dtype=np.int32)
    p0 = L.ep_plan(2, 0, counts)
    assert p0["first_expert"] == 0 and p0["local_experts"] == 3
    assert p0["send_counts"].tolist() == [3, 7] and p0["send_offsets"].tolist() == [0, 3]
    assert p0["recv_counts"].tolist() == [3, 6] and p0["recv_offsets"].tolist() == [0, 3]
    # experts 0, 1, 2 receive 3, 5, 1 rows -> padded to 128 each
    assert p0["local_offsets"].tolist() == [0, 3, 8, 9]
    assert p0["local_padded_offsets"].tolist() == [0, 128, 256, 384]
    # blocks (source, expert): (0,0) 2 rows, (0,1) 0, (0,2) 1, (1,0) 1, (1,1) 5, (1,2) 0
    assert p0["block_rows"].tolist() == [2, 0, 1, 1, 5, 0]
    assert p0["block_src"].tolist() == [0, 2, 2, 3, 4, 9]
    assert p0["block_dst"].tolist() == [0, 128, 256, 2, 128, 257]   # an empty block sits where it would start
    p1 = L.ep_plan(2, 1, counts)
    assert p1["first_expert"] == 3 and p1["local_experts"] == 2
    assert p1["send_counts"].tolist() == [6, 2] and p1["recv_counts"].tolist() == [7, 2]


def test_ep_plan_rejects_bad_arguments():
    sys.path.insert(0, ROOT)
    import latentmoe_fwd_b200 as L
    with pytest.raises(L.LmoeError):
        L.ep_plan(3, 0, np.zeros((3, 2), dtype=np.int32))          # more ranks than experts
    with pytest.raises(L.LmoeError):
        L.ep_plan(2, 0, -np.ones((2, 4), dtype=np.int32))          # negative counts


def _owner_first(G, N, h):
    base, extra = N // G, N % G
    return h * base + min(h, extra), base + (1 if h < extra else 0)


@pytest.mark.parametrize("G,N", [(2, 8), (3, 10), (4, 4)])
def test_slot_bases_follow_the_ownership_and_padded_layout(G, N):
    # written out here from the ownership rule and the padded expert-grouped
    # layout: owner h's expert e starts at the sum of its earlier experts'
    # totals (over all sources) rounded up to 128, and rank r's rows for e
    # follow those of ranks < r
    L = pytest.importorskip("latentmoe_fwd_b200")
    rng = np.random.default_rng(G * 100 + N)
    counts = rng.integers(0, 300, size=(G, N)).astype(np.int32)
    counts[0, 1] = 0
    for r in range(G):
        owner, base = L.ep_slot_bases(G, r, counts)
        for h in range(G):
            f0, nl = _owner_first(G, N, h)
            poff = 0
            for e in range(f0, f0 + nl):
                assert owner[e] == h
                assert base[e] == poff + counts[:r, e].sum()
                poff += -(-int(counts[:, e].sum()) // 128) * 128
        # the same rows as the plan's (source r, local expert) blocks at each owner
        for h in range(G):
            plan = L.ep_plan(G, h, counts)
            f0, nl = plan["first_expert"], plan["local_experts"]
            for el in range(nl):
                assert base[f0 + el] == plan["block_dst"][r * nl + el]


def test_slot_bases_reject_bad_arguments():
    sys.path.insert(0, ROOT)
    import latentmoe_fwd_b200 as L
    with pytest.raises(L.LmoeError):
        L.ep_slot_bases(3, 0, np.zeros((3, 2), dtype=np.int32))          # more ranks than experts
    with pytest.raises(L.LmoeError):
        L.ep_slot_bases(2, 0, -np.ones((2, 4), dtype=np.int32))          # negative counts
    with pytest.raises(L.LmoeError):
        L.ep_slot_bases(2, 2, np.zeros((2, 4), dtype=np.int32))          # rank out of range
