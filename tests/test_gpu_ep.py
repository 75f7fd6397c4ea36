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
