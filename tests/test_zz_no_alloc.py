"""lmoe_permute_noalloc: the permutation for callers that cannot allocate
device memory (it uses a fixed scratch array inside the library instead of a
caller workspace). Its results must equal lmoe_permute's, bit for bit, on
consecutive calls -- the shared scratch keeps the previous call's contents,
so the second call checks that nothing stale leaks into the next result.

Cases: BF16 rows with gates; NVFP4 rows (packed codes) with their block
scales re-laid to the MMA-tiled layout; and routings with out-of-range expert
indices, which both entry points leave out of every output.

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


def _sf_offsets(prow, ncols):
    """Byte offsets of scale (r, j) of padded row r in the MMA-tiled layout."""
    g64 = (ncols + 63) // 64
    r = prow[:, None].astype(np.int64)
    j = np.arange(ncols // 16, dtype=np.int64)[None, :]
    return ((r >> 7) * g64 + (j >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (j & 3)


@pytest.mark.parametrize("bad_slots", [0, 5])
def test_noalloc_permute_nvfp4_scales_and_out_of_range_slots(bad_slots):
    """Packed NVFP4 rows with row-major scales, gathered to padded rows with
    MMA-tiled scales, on two calls in a row; with bad_slots > 0 a few expert
    indices are out of range ([N, N + 3) and negative): both entry points leave
    those slots out, so offsets[N] counts only the in-range slots."""
    T, N, K, ncols = 1500, 64, 6, 256
    row_bytes = ncols // 2
    for call, seed in enumerate((21, 22)):
        rng = np.random.default_rng(seed)
        idx_np = _routing(T, N, K, seed)
        if bad_slots:
            flat = idx_np.reshape(-1)
            pos = rng.choice(flat.size, size=bad_slots, replace=False)
            flat[pos] = np.array([N, N + 2, -1, N + 1, -5][:bad_slots], dtype=np.int32)
        idx = torch.from_numpy(idx_np).cuda()
        codes = torch.from_numpy(rng.integers(0, 256, size=(T, row_bytes), dtype=np.uint8)).cuda()
        sf = torch.from_numpy(rng.integers(0, 127, size=(T, ncols // 16), dtype=np.uint8)).cuda()
        cfg = L.config(T=T, d=ncols, l=ncols, N=N, K=K, m=8)
        P = L.padded_rows(cfg)
        sf_bytes = ((P + 127) // 128) * ((ncols + 63) // 64) * 512
        outs = []
        for which in ("ws", "noalloc"):
            i32 = lambda n: torch.full((n,), -7, dtype=torch.int32, device="cuda")
            o = dict(offsets=i32(N + 1), perm_src=i32(T * K), inv_perm=i32(T * K), poff=i32(N + 1),
                     prow=torch.zeros((P, row_bytes), dtype=torch.uint8, device="cuda"),
                     psf=torch.zeros(sf_bytes, dtype=torch.uint8, device="cuda"))
            if which == "ws":
                ws = L.workspace(cfg, L.OP_PERMUTE)
                L.permute(cfg, idx, o["offsets"], o["perm_src"], o["inv_perm"], o["poff"], codes, row_bytes,
                          o["prow"], rows_sf=sf, permuted_sf=o["psf"], ws=ws)
                st, _ = L.read_device_error(ws)
                assert st == (L.ERR_DEVICE_BOUNDS if bad_slots else L.OK)
            else:
                L.permute_noalloc(cfg, idx, o["offsets"], o["perm_src"], o["inv_perm"], o["poff"], codes,
                                  row_bytes, o["prow"], rows_sf=sf, permuted_sf=o["psf"])
                torch.cuda.synchronize()
            outs.append({k: v.cpu().numpy() for k, v in o.items()})
        ref, got = outs
        n_in = int(np.sum((idx_np >= 0) & (idx_np < N)))
        assert ref["offsets"][N] == n_in and np.array_equal(got["offsets"], ref["offsets"]), call
        assert np.array_equal(got["poff"], ref["poff"]), call
        assert np.array_equal(got["perm_src"][:n_in], ref["perm_src"][:n_in]), call
        ok = ((idx_np >= 0) & (idx_np < N)).reshape(-1)
        assert np.array_equal(got["inv_perm"][ok], ref["inv_perm"][ok]), call
        # real padded rows of the in-range slots, their codes and every scale of them
        e = idx_np.reshape(-1)[ok].astype(np.int64)
        prow = ref["inv_perm"][ok] - ref["offsets"][e] + ref["poff"][e]
        assert np.array_equal(got["prow"][prow], ref["prow"][prow]), call
        offs = _sf_offsets(prow, ncols)
        assert np.array_equal(got["psf"][offs], ref["psf"][offs]), call
        # and the gathered scales are the source rows' scales
        src_tok = np.nonzero(ok)[0] // K
        assert np.array_equal(ref["psf"][offs], sf.cpu().numpy()[src_tok]), call
