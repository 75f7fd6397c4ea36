"""lmoe_permute_noalloc: the permutation for callers that cannot allocate
device memory (it uses a fixed scratch array inside the library instead of a
caller workspace). Its results must equal lmoe_permute's, bit for bit, on
consecutive calls -- the shared scratch keeps the previous call's contents,
so the second call checks that nothing stale leaks into the next result.

This file is collected last so that a run stopping at its first failure has
already run every other test."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

L = pytest.importorskip("latentmoe_fwd_b200")


def _routing(T, N, K, seed):
    rng = np.random.default_rng(seed)
    return np.argsort(rng.random((T, N)), axis=1)[:, :K].astype(np.int32)


def _outputs(T, N, K, row_elems):
    i32 = lambda n: torch.full((n,), -7, dtype=torch.int32, device="cuda")
    cfg = L.config(T=T, d=row_elems, l=row_elems, N=N, K=K, m=8)
    P = L.padded_rows(cfg)
    return cfg, dict(offsets=i32(N + 1), perm_src=i32(T * K), inv_perm=i32(T * K), poff=i32(N + 1),
                     prow=torch.zeros((P, row_elems), dtype=torch.bfloat16, device="cuda"),
                     pgate=torch.zeros(P, dtype=torch.float32, device="cuda"))


@pytest.mark.parametrize("shape", [(3000, 512, 22), (4096, 128, 6)])
def test_noalloc_permute_matches_workspace_permute_on_two_calls(shape):
    T, N, K = shape
    row_elems = 64
    for call, seed in enumerate((11, 12)):          # two calls in a row, different routings
        idx = torch.from_numpy(_routing(T, N, K, seed)).cuda()
        rows = torch.randn((T, row_elems), device="cuda").to(torch.bfloat16)
        w = torch.rand((T, K), device="cuda")
        cfg, ref = _outputs(T, N, K, row_elems)
        ws = L.workspace(cfg, L.OP_PERMUTE)
        L.permute(cfg, idx, ref["offsets"], ref["perm_src"], ref["inv_perm"], ref["poff"], rows, row_elems * 2,
                  ref["prow"], topk_w=w, perm_gate=ref["pgate"], ws=ws)
        assert L.read_device_error(ws)[0] == L.OK
        _, got = _outputs(T, N, K, row_elems)
        L.permute_noalloc(cfg, idx, got["offsets"], got["perm_src"], got["inv_perm"], got["poff"], rows,
                          row_elems * 2, got["prow"], topk_w=w, perm_gate=got["pgate"])
        torch.cuda.synchronize()
        for key in ("offsets", "perm_src", "inv_perm", "poff"):
            assert torch.equal(got[key], ref[key]), (call, key)
        n = int(ref["poff"][-1].item())
        # padded rows hold only what was gathered; compare the rows of real slots
        real = torch.zeros(n, dtype=torch.bool, device="cuda")
        flat = idx.reshape(-1).long()
        pr = ref["inv_perm"].long() - ref["offsets"].long()[flat] + ref["poff"].long()[flat]
        real[pr] = True
        assert torch.equal(got["prow"][:n][real], ref["prow"][:n][real]), call
        assert torch.equal(got["pgate"][:n][real], ref["pgate"][:n][real]), call


def test_noalloc_permute_rejects_problems_beyond_its_scratch():
    T, N, K = 300000, 1024, 8                    # (ceil(T*K/8192) + 1) * N counters > 131072
    cfg = L.config(T=T, d=8, l=8, N=N, K=K, m=8)
    dummy = torch.zeros(16, dtype=torch.int32, device="cuda")
    with pytest.raises(L.LmoeError) as e:
        L.permute_noalloc(cfg, dummy, dummy, dummy, dummy, dummy)
    assert e.value.status == L.ERR_WORKSPACE
