"""Cases run under the bounds-checking debug build (liblmoe_checks.so).

Run by tests/test_gpu_checks.py in a child process with LMOE_LIBRARY set, so
this process loads the debug build instead of the release one:

1. small layer forwards (BF16 latent layers on single-CTA and CTA-pair
   tiles, an identity layer with shared experts, NVFP4, fp32) against the
   oracle, with the same bars as the release build's tests;
2. lmoe_expert_ffn (BF16 and NVFP4) given offsets whose expert claims more
   rows than its padded range holds: the debug build records
   LMOE_ERR_DEVICE_BOUNDS and skips that expert, the other experts' rows are
   still right, and the context stays usable;
3. lmoe_combine given a slot whose row lies past the padded rows: the debug
   build leaves that slot out of the sum.
Every buffer these cases hand over has room for the rows a bad offset names,
so no access leaves memory the test owns even where a check were missing.
"""
import os
import sys

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))
sys.path.insert(0, HERE)

import latentmoe_fwd_b200 as L  # noqa: E402
import lmoe_inputs as LI  # noqa: E402
from oracle import lmoe_oracle as O  # noqa: E402
from gpu_util import DevLayer, as_f64, bf16_parity, rel_max_err, to_dev  # noqa: E402


def forward_case(wl, tol):
    inp = LI.make_inputs(wl)
    dev = DevLayer(wl, inp)
    out = as_f64(dev.forward())
    ref = O.forward(wl, inp)
    gidx, _, _ = dev.route()
    same = np.all(gidx == ref["idx"], axis=1)
    near = O.near_tie_tokens(ref["logits"], wl.K)
    assert np.all(same | near)
    keep = same
    if wl.dtype == "nvfp4":   # allow the documented z-rounding near-ties, as the release tests do
        from test_gpu_nvfp4 import nvfp4_token_errors
        toks = np.nonzero(keep)[0]
        e, _, _ = nvfp4_token_errors(wl, inp, out, gidx, toks, tol)
        print(f"checks build: {wl.name} T={wl.T}: err {e.max():.3e} * RMS")
        assert e.max() <= tol, (wl.name, e.max())
        return
    if wl.dtype == "f32":
        err = rel_max_err(out[keep], ref["out"][keep])
    else:
        err, _ = bf16_parity(out[keep], ref["out_unrounded"][keep], ref["out"][keep])
    print(f"checks build: {wl.name} T={wl.T}: err {err:.3e} * RMS")
    assert err <= tol, (wl.name, err)


def bad_offsets_case(nvfp4: bool):
    wl = LI.reduced("ultra_nvfp4" if nvfp4 else "ultra_decode", T=300, d=512, l=256, N=8, K=2, m=256)
    inp = LI.make_inputs(wl)
    dev = DevLayer(wl, inp)
    cfg = dev.cfg
    T, K, N, l = wl.T, wl.K, wl.N, wl.l
    P = L.padded_rows(cfg)
    idx = torch.from_numpy(O.route_topk(O.router_logits(O.from_bf16_bits(inp["x"]),
                                                        O.from_bf16_bits(inp["w_router"])), K)[0]).cuda()
    i32 = lambda n: torch.zeros(n, dtype=torch.int32, device="cuda")
    offsets, poff, src, inv = i32(N + 1), i32(N + 1), i32(T * K), i32(T * K)
    rng = np.random.default_rng(5)
    z = torch.from_numpy(LI.bf16_bits(rng.standard_normal((T, l))).view(np.int16)).view(torch.bfloat16).cuda()
    slack = 2 * P                                     # room for any row a bad offset can name
    ws = L.workspace(cfg, L.OP_PERMUTE)
    if nvfp4:
        from gpu_util import quantize_dev
        codes, sf, g = quantize_dev(z, T, l)
        zp = torch.zeros((slack, l // 2), dtype=torch.uint8, device="cuda")
        zsf = torch.zeros(slack * l // 16, dtype=torch.uint8, device="cuda")
        L.permute(cfg, idx, offsets, src, inv, poff, codes, l // 2, zp, rows_sf=sf, permuted_sf=zsf, ws=ws)
    else:
        zp = torch.zeros((slack, l), dtype=torch.bfloat16, device="cuda")
        zsf, g = None, None
        L.permute(cfg, idx, offsets, src, inv, poff, z, l * 2, zp, ws=ws)
    assert L.read_device_error(ws)[0] == L.OK
    y_ok = torch.zeros((slack, l), dtype=torch.bfloat16, device="cuda")
    ws2 = L.workspace(L.config(T=2 * T, d=wl.d, l=l, N=N, K=K, m=wl.m, expert=cfg.expert), L.OP_EXPERT_FFN)
    L.expert_ffn(cfg, dev.w, zp, zsf, g, offsets, poff, None, y_ok, ws2)
    assert L.read_device_error(ws2)[0] == L.OK
    # expert 1 claims 200 rows more than its padded range holds
    bad = offsets.clone()
    bad[2:] += 200
    y_bad = torch.zeros_like(y_ok)
    L.expert_ffn(cfg, dev.w, zp, zsf, g, bad, poff, None, y_bad, ws2)
    st, info = L.read_device_error(ws2)
    print(f"checks build: bad offsets ({'NVFP4' if nvfp4 else 'BF16'}): status {L.status_string(st)} info {info:#x}")
    assert st == L.ERR_DEVICE_BOUNDS
    off = offsets.cpu().numpy()
    po = poff.cpu().numpy()
    r0 = slice(int(po[0]), int(po[0] + off[1] - off[0]))   # expert 0's rows are unaffected
    assert torch.equal(y_bad[r0], y_ok[r0])
    assert torch.count_nonzero(y_bad[int(po[1]):int(po[2])]) == 0   # the bad expert was skipped
    dev.forward()                                     # the context is still usable


def combine_case():
    T, K, N, l = 64, 2, 4, 64
    cfg = L.config(T=T, d=l, l=l, N=N, K=K, m=64)
    idx = torch.from_numpy(np.stack([np.arange(T) % N, (np.arange(T) + 1) % N], 1).astype(np.int32)).cuda()
    i32 = lambda n: torch.zeros(n, dtype=torch.int32, device="cuda")
    offsets, poff, src, inv = i32(N + 1), i32(N + 1), i32(T * K), i32(T * K)
    ws = L.workspace(cfg, L.OP_PERMUTE)
    L.permute(cfg, idx, offsets, src, inv, poff, ws=ws)
    P = L.padded_rows(cfg)
    y = torch.randn((4 * P, l), device="cuda").to(torch.bfloat16)
    c_ok = torch.empty((T, l), dtype=torch.bfloat16, device="cuda")
    L.combine(cfg, y, idx, inv, offsets, poff, None, c_ok)
    bad_inv = inv.clone()
    bad_inv[5 * K + 1] += 2 * P                       # token 5's second slot points past the padded rows
    c_bad = torch.empty_like(c_ok)
    L.combine(cfg, y, idx, bad_inv, offsets, poff, None, c_bad)
    torch.cuda.synchronize()
    e0 = int(idx[5, 0])
    row0 = int(inv[5 * K]) - int(offsets[e0]) + int(poff[e0])
    assert torch.equal(c_bad[5], y[row0])             # only the in-range slot is summed
    keep = torch.ones(T, dtype=torch.bool)
    keep[5] = False
    assert torch.equal(c_bad[keep.cuda()], c_ok[keep.cuda()])
    print("checks build: combine left out the out-of-range slot")


def main():
    assert os.path.basename(L.LIB_PATH) == "liblmoe_checks.so", L.LIB_PATH
    torch.cuda.set_device(0)
    forward_case(LI.reduced("ultra_decode", T=700, d=512, l=256, N=64, K=8, m=384), 2e-2)   # CTA pairs
    forward_case(LI.reduced("ultra_decode", T=32, d=512, l=256, N=64, K=8, m=384), 2e-2)    # weight-major
    forward_case(LI.reduced("std_moe_bf16", T=300, d=512, l=512, N=8, K=2, m=320, n_shared=2, m_shared=192), 2e-2)
    forward_case(LI.reduced("ultra_nvfp4", T=256, d=512, l=256, N=8, K=2, m=256), 8e-2)
    forward_case(LI.WORKLOADS["tiny_f32"], 1e-4)
    bad_offsets_case(nvfp4=False)
    bad_offsets_case(nvfp4=True)
    combine_case()
    print("CHECKS_OK")


if __name__ == "__main__":
    main()
