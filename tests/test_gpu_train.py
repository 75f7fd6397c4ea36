"""The NVFP4 training recipe's pieces on the GPU (row f4), through the C ABI,
against the backward oracle (oracle/lmoe_backward.py):

* lmoe_nvfp4_quantize_ex bit-exact: stochastic rounding with Philox-4x32-10
  uniforms drawn on the device at the oracle's counters, the 16-point random
  Hadamard transform along the tokens with a transposed output, round to
  nearest, and 16 x 16 blocks of a transposed weight;
* dgrad and wgrad of one linear layer under the recipe (quantiser + the
  block-scaled tcgen05 GEMM) against nvfp4_linear_backward;
* the routed experts' weight and input gradients of a small layer against
  backward_nvfp4.
"""
import numpy as np
import pytest
import torch

import lmoe_inputs as LI
from oracle import lmoe_backward as B
from oracle import lmoe_oracle as O

pytestmark = pytest.mark.gpu

L = pytest.importorskip("latentmoe_fwd_b200")
from gpu_util import to_dev  # noqa: E402

SIGNS = np.array([1, -1, -1, 1, 1, 1, -1, 1, -1, 1, 1, -1, -1, -1, 1, 1], dtype=np.float64)
SIGN_BITS = int(sum(1 << i for i in range(16) if SIGNS[i] < 0))


def _quantize_ex(x_bits, rows, cols, flags, seed=0, stream=0, layout=L.SF_ROWMAJOR):
    tr = bool(flags & L.QX_TRANSPOSE)
    R, C = (cols, rows) if tr else (rows, cols)
    codes = torch.empty((R, C // 2), dtype=torch.uint8, device="cuda")
    sf = torch.zeros((R, C // 16), dtype=torch.uint8, device="cuda")
    g = torch.empty(1, dtype=torch.float32, device="cuda")
    L.nvfp4_quantize_ex(to_dev(x_bits, "bf16"), L.BF16, rows, cols, flags, SIGN_BITS, seed, stream, None, codes, sf,
                        g, layout)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), sf.cpu().numpy(), float(g.item())


def _data(rows, cols, seed):
    rng = np.random.default_rng(seed)
    v = rng.standard_normal((rows, cols)) * np.exp(rng.uniform(-3, 3, size=(rows, 1)))
    return LI.bf16_bits(v)


@pytest.mark.parametrize("rows,cols", [(16, 16), (48, 160), (256, 512)])
def test_stochastic_rounding_bit_exact(rows, cols):
    bits = _data(rows, cols, rows + cols)
    X = O.from_bf16_bits(bits)
    seed, stream = 0x1234_5678_9ABC, 7
    codes, sf, g = _quantize_ex(bits, rows, cols, L.QX_SR, seed, stream)
    u = B.sr_uniforms(rows * cols, seed, stream).reshape(rows, cols)
    rc, rsf, rg = B.nvfp4_quantize_sr(X, u)
    assert g == np.float32(rg)
    assert np.array_equal(sf, rsf)
    assert np.array_equal(codes, rc)
    # and it differs from round-to-nearest somewhere (the uniforms matter)
    nc, _, _ = O.nvfp4_quantize(X)
    assert not np.array_equal(codes, nc)


@pytest.mark.parametrize("sr", [False, True])
def test_rht_along_tokens_transposed_bit_exact(sr):
    T, n = 64, 96                                     # tokens x features (a wgrad operand)
    bits = _data(T, n, 11)
    X = O.from_bf16_bits(bits)
    flags = L.QX_TRANSPOSE | L.QX_RHT | (L.QX_SR if sr else 0)
    codes, sf, g = _quantize_ex(bits, T, n, flags, seed=99, stream=3)
    Xt = B.rht(X, SIGNS, axis=0).T                    # [n, T]: transformed along the tokens
    if sr:
        u = B.sr_uniforms(n * T, 99, 3).reshape(n, T)
        rc, rsf, rg = B.nvfp4_quantize_sr(Xt, u)
    else:
        rc, rsf, rg = O.nvfp4_quantize(Xt)
    assert g == np.float32(rg)
    assert np.array_equal(sf, rsf)
    assert np.array_equal(codes, rc)


def test_transposed_weight_2d_blocks_bit_exact():
    W = _data(80, 128, 5)                             # [n_out, n_in]; dgrad reads W^T [n_in, n_out]
    codes, sf, g = _quantize_ex(W, 80, 128, L.QX_TRANSPOSE, layout=L.SF_ROWMAJOR | L.SF_BLOCK_16X16)
    rc, rsf, rg = O.nvfp4_quantize_2d(O.from_bf16_bits(W).T)
    assert g == np.float32(rg)
    assert np.array_equal(sf, rsf) and np.array_equal(codes, rc)
    # 16 x 16 blocks quantise W and W^T alike
    wc, wsf, _ = O.nvfp4_quantize_2d(O.from_bf16_bits(W))
    assert np.array_equal(O.nvfp4_dequantize(rc, rsf, rg), O.nvfp4_dequantize(wc, wsf, rg).T)


@pytest.mark.parametrize("layout", ["rowmajor", "tiled"])
def test_ragged_2d_blocks_bit_exact(layout):
    # 40 rows: the last 16 x 16 blocks hold 8 rows (the rest count as 0)
    W = _data(40, 96, 9)
    lay = (L.SF_ROWMAJOR if layout == "rowmajor" else L.SF_MMA_TILED) | L.SF_BLOCK_16X16
    if layout == "tiled":
        codes = torch.empty((40, 48), dtype=torch.uint8, device="cuda")
        sf = torch.zeros((40 + 127) // 128 * ((96 + 63) // 64) * 512, dtype=torch.uint8, device="cuda")
        g = torch.empty(1, dtype=torch.float32, device="cuda")
        L.nvfp4_quantize_ex(to_dev(W, "bf16"), L.BF16, 40, 96, 0, SIGN_BITS, 0, 0, None, codes, sf, g, lay)
        torch.cuda.synchronize()
        codes, sf, g = codes.cpu().numpy(), sf.cpu().numpy(), float(g.item())
        rc, rsf, rg = O.nvfp4_quantize_2d(O.from_bf16_bits(W))
        assert g == np.float32(rg) and np.array_equal(codes, rc)
        r, j = np.arange(40)[:, None], np.arange(96 // 16)[None, :]   # the documented MMA-tiled offsets
        off = ((r >> 7) * ((96 + 63) // 64) + (j >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (j & 3)
        assert np.array_equal(sf[off], rsf)
        return
    codes, sf, g = _quantize_ex(W, 40, 96, 0, layout=lay)
    rc, rsf, rg = O.nvfp4_quantize_2d(O.from_bf16_bits(W))
    assert g == np.float32(rg) and np.array_equal(sf, rsf) and np.array_equal(codes, rc)


@pytest.mark.parametrize("groups,rows,cols", [(1, 128, 128), (3, 256, 384)])
def test_transpose_2d_equals_quantising_the_transpose(groups, rows, cols):
    # W^T with 16 x 16 blocks quantises to W's codes and scales transposed
    lay = L.SF_MMA_TILED | L.SF_BLOCK_16X16
    Ws = [_data(rows, cols, 40 + g) for g in range(groups)]
    codes = torch.empty((groups, rows, cols // 2), dtype=torch.uint8, device="cuda")
    sf = torch.zeros((groups, rows * cols // 16), dtype=torch.uint8, device="cuda")
    ref_c = torch.empty((groups, cols, rows // 2), dtype=torch.uint8, device="cuda")
    ref_s = torch.zeros((groups, rows * cols // 16), dtype=torch.uint8, device="cuda")
    gl = torch.empty(2 * groups, dtype=torch.float32, device="cuda")
    for g, W in enumerate(Ws):
        x = to_dev(W, "bf16")
        L.nvfp4_quantize_ex(x, L.BF16, rows, cols, 0, 0, 0, 0, None, codes[g], sf[g], gl[2 * g:], lay)
        L.nvfp4_quantize_ex(x, L.BF16, rows, cols, L.QX_TRANSPOSE, 0, 0, 0, None, ref_c[g], ref_s[g],
                            gl[2 * g + 1:], lay)
    ct = torch.full_like(ref_c, 0xAA)
    st = torch.full_like(ref_s, 0xAA)
    L.nvfp4_transpose_2d(codes, sf, groups, rows, cols, ct, st)
    torch.cuda.synchronize()
    g = gl.cpu().numpy()
    assert np.array_equal(g[0::2], g[1::2])
    assert torch.equal(ct, ref_c) and torch.equal(st, ref_s)


def test_plain_mode_equals_nvfp4_quantize():
    bits = _data(130, 64, 2)
    codes, sf, g = _quantize_ex(bits, 130, 64, 0)
    rc, rsf, rg = O.nvfp4_quantize(O.from_bf16_bits(bits))
    assert g == np.float32(rg) and np.array_equal(sf, rsf) and np.array_equal(codes, rc)


def test_stochastic_rounding_of_midpoint_values():
    """Values that land half way between two E2M1 grid points after scaling
    round up exactly when u < 1/2, so these codes follow the top bit of each
    Philox word: the device's draws match the oracle's generator word for word."""
    rows, cols = 4, 64
    v = np.full((rows, cols), 0.75)                   # amax 0.75 -> s_g, scale: v / sc between 0.5 and 1
    v[:, 0] = 6.0 * 0.75 / 0.75                       # give each block an amax that maps to 6 exactly
    bits = LI.bf16_bits(v)
    X = O.from_bf16_bits(bits)
    codes, sf, g = _quantize_ex(bits, rows, cols, L.QX_SR, seed=42, stream=1)
    u = B.sr_uniforms(rows * cols, 42, 1).reshape(rows, cols)
    rc, rsf, rg = B.nvfp4_quantize_sr(X, u)
    assert np.array_equal(codes, rc) and np.array_equal(sf, rsf)


def _q_dev(x_dev, rows, cols, flags, seed=0, stream=0, block2d=False):
    """lmoe_nvfp4_quantize_ex into MMA-tiled scales (the GEMM's operand layout)."""
    tr = bool(flags & L.QX_TRANSPOSE)
    R, C = (cols, rows) if tr else (rows, cols)
    codes = torch.empty((R, C // 2), dtype=torch.uint8, device="cuda")
    sf = torch.zeros((((R + 127) // 128) * 128 * ((C + 63) // 64) * 4,), dtype=torch.uint8, device="cuda")
    g = torch.empty(1, dtype=torch.float32, device="cuda")
    layout = L.SF_MMA_TILED | (L.SF_BLOCK_16X16 if block2d else 0)
    L.nvfp4_quantize_ex(x_dev, L.BF16, rows, cols, flags, SIGN_BITS, seed, stream, None, codes, sf, g, layout)
    return codes, sf, g


def _gemm_dev(a, a_rows, b, cols, k):
    """Plain (one-group) block-scaled GEMM: BF16 [a_rows][cols] = A . B^T."""
    out = torch.empty((a_rows, cols), dtype=torch.bfloat16, device="cuda")
    offs = torch.tensor([0, a_rows], dtype=torch.int32, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    L.nvfp4_gemm(1, offs, offs, a_rows, a[0], a[1], a[2], 0, b[0], b[1], b[2], cols, k, None, out, cols, ws)
    st, info = L.read_device_error(ws)
    assert st == L.OK, (L.status_string(st), hex(info))
    return out.float().cpu().numpy().astype(np.float64)


def test_linear_layer_dgrad_and_wgrad_match_the_oracle():
    """dX = Q_sr(dY) Q_2d(W) and dW = Q_sr(RHT(dY)^T) Q_rn(RHT(X)^T)^T on the GPU
    (quantiser + block-scaled tcgen05 GEMM) against nvfp4_linear_backward."""
    from gpu_util import bf16_parity
    T, n_in, n_out = 256, 256, 512
    rng = np.random.default_rng(8)
    Xb = LI.bf16_bits(rng.standard_normal((T, n_in)))
    Wb = LI.bf16_bits(rng.standard_normal((n_out, n_in)) / np.sqrt(n_in))
    dYb = LI.bf16_bits(rng.standard_normal((T, n_out)) * 0.01)
    X, W, dY = (O.from_bf16_bits(b) for b in (Xb, Wb, dYb))
    seed, s_dgrad, s_wgrad = 2026, 10, 11
    x, w, dy = (to_dev(b, "bf16") for b in (Xb, Wb, dYb))
    # dgrad: contraction over n_out
    a = _q_dev(dy, T, n_out, L.QX_SR, seed, s_dgrad)
    b = _q_dev(w, n_out, n_in, L.QX_TRANSPOSE, block2d=True)          # W^T [n_in][n_out], 16 x 16 blocks
    dX = _gemm_dev(a, T, b, n_in, n_out)
    # wgrad: contraction over the tokens, both operands transformed along them
    a = _q_dev(dy, T, n_out, L.QX_TRANSPOSE | L.QX_RHT | L.QX_SR, seed, s_wgrad)
    b = _q_dev(x, T, n_in, L.QX_TRANSPOSE | L.QX_RHT)
    dW = _gemm_dev(a, n_out, b, n_in, T)
    ref = B.nvfp4_linear_backward(X, W, dY, SIGNS, B.sr_uniforms(T * n_out, seed, s_dgrad).reshape(T, n_out),
                                  B.sr_uniforms(n_out * T, seed, s_wgrad).reshape(n_out, T))
    for name, got, exact in (("dX", dX, ref["dX"]), ("dW", dW, ref["dW"])):
        excess, raw = bf16_parity(got, exact, O.round_bf16(exact))
        print(f"linear backward {name}: excess {excess:.3e} * RMS, raw {raw:.3e} * RMS")
        assert excess <= 2e-2, name
    # the quantised gradients differ from the exact ones (the recipe's rounding is visible)
    exact = B.nvfp4_linear_backward(X, W, dY, SIGNS, None, None, quantize=False)
    rel = np.sqrt(np.mean((dW - exact["dW"]) ** 2) / np.mean(exact["dW"] ** 2))
    assert 1e-3 < rel < 0.5


@pytest.mark.parametrize("T,N,K,zero_expert", [(160, 4, 2, False), (96, 8, 3, True)])
def test_routed_experts_backward_matches_the_oracle(T, N, K, zero_expert):
    """lmoe_expert_backward_nvfp4 (recomputed NVFP4 forward, SR dgrad, RHT +
    SR wgrad for both expert GEMMs, every step a kernel of the library) against
    the oracle's routed_experts_backward_nvfp4 on the same NVFP4 latent rows,
    routing, gates and upstream gradient.

    The GPU forms a stochastic quantiser's input (dh = dA * 2 relu(h)) with
    fp32 GEMMs where the oracle is exact, so an element whose value sits
    within that rounding of its uniform's threshold takes the other grid
    neighbour. The tensor cores' fp32 accumulation is off by up to ~2^-13 of
    the L2 norm of a dot product's terms (the window of the z-rounding ties),
    so about 1e-4 of the elements flip: a few per expert here. In dz and dgate
    such a flip is one term of a long sum; in a weight gradient it moves one
    whole row (a flip in the gradient operand) or column (in the activation
    operand) of that expert's dW by one quantisation step times the other
    operand, up to several tenths of RMS(dW). So: dz and dgate within the NVFP4
    forward's 8e-2 * RMS bar beyond half a BF16 step everywhere; dW within it
    outside at most eight such lines per expert (and 2% of its elements); every
    output within 1e-2 in
    relative Frobenius norm, and at least 5x closer to the oracle than the
    oracle is to the unquantised gradient (dz, dW)."""
    from gpu_util import bf16_parity, quantize_dev
    l = m = 256
    rng = np.random.default_rng(T * 7 + N)
    zb = LI.bf16_bits(rng.standard_normal((T, l)))
    w1b = LI.bf16_bits(rng.standard_normal((N, m, l)) / np.sqrt(l))
    w2b = LI.bf16_bits(rng.standard_normal((N, l, m)) / np.sqrt(m))
    dcb = LI.bf16_bits(rng.standard_normal((T, l)) * 0.05)
    logits = rng.standard_normal((T, N))
    if zero_expert:
        logits[:, N - 1] = -50.0                            # an expert no token reaches
    idx, gates = O.route_topk(logits, K)
    s_a = float(np.float32(20.0 / 2688.0))                  # static global scale of a
    seed = 0x5EED
    z, w1, w2, dc = (O.from_bf16_bits(b) for b in (zb, w1b, w2b, dcb))

    # oracle, on the NVFP4 latent rows the GPU quantiser produces (bit-exact, pinned elsewhere)
    zq, _ = O.nvfp4_fake_quant(z)
    ref = B.routed_experts_backward_nvfp4(zq, w1, w2, idx, gates, dc, SIGNS, seed, s_a)

    # device: quantise z, permute rows (NVFP4 codes + tiled scales) and gates
    cfg = L.config(T=T, d=l, l=l, N=N, K=K, m=m, expert=L.NVFP4)
    P = L.padded_rows(cfg)
    codes, sf, zgs = quantize_dev(to_dev(zb, "bf16"), T, l)
    i32 = lambda n: torch.empty(n, dtype=torch.int32, device="cuda")
    offsets, poff, perm_src, inv_perm = i32(N + 1), i32(N + 1), i32(T * K), i32(T * K)
    zp = torch.zeros((P, l // 2), dtype=torch.uint8, device="cuda")
    zp_sf = torch.zeros(P * l // 16, dtype=torch.uint8, device="cuda")
    pgate = torch.zeros(P, dtype=torch.float32, device="cuda")
    idx_d = torch.from_numpy(idx.astype(np.int32)).cuda()
    gates_d = torch.from_numpy(gates.astype(np.float32)).cuda()
    ws = L.workspace(cfg, L.OP_PERMUTE)
    L.permute(cfg, idx_d, offsets, perm_src, inv_perm, poff, codes, l // 2, zp, sf, zp_sf, gates_d, pgate, ws=ws)
    assert L.read_device_error(ws)[0] == L.OK
    # each padded row's upstream gradient: dc of its token
    counts = np.bincount(idx.reshape(-1), minlength=N).astype(np.int32)
    off_h, poff_h, src_h = offsets.cpu().numpy(), poff.cpu().numpy(), perm_src.cpu().numpy()
    row_of = np.empty(T * K, dtype=np.int64)                # slot f -> padded row
    for r, f in enumerate(src_h):
        e = idx.reshape(-1)[f]
        row_of[f] = r - off_h[e] + poff_h[e]
    dy_pad = np.zeros((P, l), dtype=np.float32)
    dy_pad[row_of] = dc[np.arange(T * K) // K]
    dy = to_dev(dy_pad, "f32")
    a_g = torch.tensor([s_a], dtype=torch.float32, device="cuda")
    dz = torch.zeros((P, l), dtype=torch.bfloat16, device="cuda")
    dgate = torch.zeros(P, dtype=torch.float32, device="cuda")
    dw1 = torch.empty((N, m, l), dtype=torch.bfloat16, device="cuda")
    dw2 = torch.empty((N, l, m), dtype=torch.bfloat16, device="cuda")
    bws = L.expert_backward_nvfp4(cfg, counts, offsets, poff, zp, zp_sf, zgs, to_dev(w1b, "bf16"),
                                  to_dev(w2b, "bf16"), a_g, pgate, dy, seed, SIGN_BITS, dz, dgate, dw1, dw2)
    st, info = L.read_device_error(bws)
    assert st == L.OK, (L.status_string(st), hex(info))

    # back to tokens: dz summed over each token's slots, dgate per (token, k)
    dz_rows = dz.float().cpu().numpy().astype(np.float64)
    dz_tok = np.zeros((T, l))
    np.add.at(dz_tok, np.arange(T * K) // K, dz_rows[row_of])
    dgate_tk = dgate.cpu().numpy().astype(np.float64)[row_of].reshape(T, K)
    got = dict(dz=dz_tok, dgate=dgate_tk, dw1=dw1.float().cpu().numpy().astype(np.float64),
               dw2=dw2.float().cpu().numpy().astype(np.float64))
    exact = B.routed_experts_backward_nvfp4(zq, w1, w2, idx, gates, dc, SIGNS, seed, s_a, quantize=False)
    from gpu_util import bf16_ulp
    for name in ("dz", "dgate", "dw1", "dw2"):
        g, r = got[name], ref[name]
        excess, raw = bf16_parity(g, r, O.round_bf16(r))
        fro = np.linalg.norm(g - r) / np.linalg.norm(r)
        qerr = np.linalg.norm(exact[name] - r) / np.linalg.norm(r)
        print(f"experts backward {name}: excess {excess:.3e} * RMS, raw {raw:.3e} * RMS, rel {fro:.3e} "
              f"(recipe vs unquantised: {qerr:.3e})")
        assert fro <= 1e-2, name
        if name in ("dz", "dgate"):
            assert excess <= 8e-2, name
        else:
            # elements beyond the bar, per expert: covered by at most two rows or two columns
            rms = np.sqrt(np.mean(O.round_bf16(r) ** 2))
            over = (np.abs(g - r) - bf16_ulp(O.round_bf16(r)) / 2) > 8e-2 * rms
            for e in range(N):
                rows, cols = np.nonzero(over[e])
                lines = min(np.unique(rows).size, np.unique(cols).size)
                if lines:
                    print(f"  {name}[{e}]: {rows.size} elements beyond the bar on {lines} line(s)")
                assert lines <= 8, (name, e)
            assert over.mean() <= 0.02, name
        if name != "dgate":
            assert fro < 0.2 * qerr, name   # far closer to the oracle than to the unquantised value
    if zero_expert:
        assert not np.any(got["dw1"][N - 1]) and not np.any(got["dw2"][N - 1])


def _weight_grad_check(name, g, r, N_groups=None):
    """The weight-gradient bar of the layer test: 1e-2 relative Frobenius error,
    and elements beyond 8e-2 * RMS (past half a BF16 step) confined to at most
    a tenth of the rows or of the columns of each expert's matrix (at least
    eight), 5% of its elements: stochastic-rounding flips, more frequent when
    an expert has few rows (each flip then weighs more)."""
    from gpu_util import bf16_ulp
    fro = np.linalg.norm(g - r) / np.linalg.norm(r)
    rms = np.sqrt(np.mean(O.round_bf16(r) ** 2))
    over = (np.abs(g - r) - bf16_ulp(O.round_bf16(r)) / 2) > 8e-2 * rms
    cap = max(8, over.shape[1] // 10, over.shape[2] // 10)
    for e in range(over.shape[0]):
        rows, cols = np.nonzero(over[e])
        assert min(np.unique(rows).size, np.unique(cols).size) <= cap, (name, e)
    assert over.mean() <= 0.05, name
    assert fro <= 1e-2, name
    return fro


@pytest.mark.parametrize("case", ["latent", "latent_shared_bias", "identity_shared"])
def test_layer_backward_matches_the_oracle(case):
    """lmoe_backward_nvfp4 (the whole layer's gradients: recomputed routing and
    NVFP4 latent rows, the routed experts under the recipe, the router, the
    latent projections and the shared experts as BF16 GEMMs) against the
    oracle's backward_nvfp4 on the same inputs. The dense gradients are BF16
    GEMMs of BF16-rounded gradient tensors: within 2e-2 * RMS beyond half a
    BF16 step (the BF16 forward's bar); dW1 and dW2 as in the expert test."""
    from gpu_util import DevLayer, bf16_parity
    if case == "latent":
        wl = LI.reduced("ultra_decode", T=160, d=512, l=256, N=8, K=2, m=256)
    elif case == "latent_shared_bias":
        wl = LI.replace(LI.reduced("ultra_zipf", T=96, d=512, l=256, N=8, K=3, m=256, n_shared=1, m_shared=128))
    else:
        wl = LI.reduced("std_moe_bf16", T=128, d=256, l=256, N=8, K=2, m=256, n_shared=2, m_shared=64)
    inp = LI.make_inputs(wl)
    p = B.params_from_inputs(wl, inp)
    rng = np.random.default_rng(11)
    doutb = LI.bf16_bits(rng.standard_normal((wl.T, wl.d)) * 0.05)
    dout = O.from_bf16_bits(doutb)
    # static global scale of a from the unquantised expert pre-activations
    x = p["x"]
    z = x if p["w_down"] is None else x @ p["w_down"].T
    amax = max(np.max(O.sq_relu(z @ p["w1"][e].T)) for e in range(wl.N))
    s_a = float(np.float32(amax / 2688.0))
    seed = 0xBEEF
    logits = O.router_logits(x, p["w_router"], p["router_bias"])
    assert not np.any(O.near_tie_tokens(logits, wl.K)), "near-tie routing in the test data"
    ref = B.backward_nvfp4(p, wl.K, dout, SIGNS, seed, a_global_scale=s_a)

    dev = DevLayer(wl, inp)
    bf = lambda *shape: torch.zeros(shape, dtype=torch.bfloat16, device="cuda")
    S, ms = wl.n_shared, wl.m_shared
    out = dict(dx=bf(wl.T, wl.d), dw_router=bf(wl.N, wl.d), dw1=bf(wl.N, wl.m, wl.l), dw2=bf(wl.N, wl.l, wl.m))
    if inp["router_bias"] is not None:
        out["drouter_bias"] = torch.zeros(wl.N, dtype=torch.float32, device="cuda")
    if not wl.identity:
        out.update(dw_down=bf(wl.l, wl.d), dw_up=bf(wl.d, wl.l))
    if S:
        out.update(dws1=bf(S, ms, wl.d), dws2=bf(S, wl.d, ms))
    g = L.grads(**out)
    a_g = torch.tensor([s_a], dtype=torch.float32, device="cuda")
    ws = L.backward_nvfp4(dev.cfg, dev.w, dev.x, to_dev(doutb, "bf16"), a_g, seed, SIGN_BITS, g)
    st, info = L.read_device_error(ws)
    assert st == L.OK, (L.status_string(st), hex(info))
    got = {k: v.float().cpu().numpy().astype(np.float64) for k, v in out.items()}
    for name in ("dx", "dw_router", "drouter_bias", "dw_down", "dw_up", "dws1", "dws2"):
        if name not in got:
            continue
        r = ref[name]
        excess, raw = bf16_parity(got[name], r, O.round_bf16(r))
        fro = np.linalg.norm(got[name] - r) / np.linalg.norm(r)
        print(f"layer backward {case} {name}: excess {excess:.3e} * RMS, raw {raw:.3e} * RMS, rel {fro:.3e}")
        assert excess <= 2e-2, name
    for name in ("dw1", "dw2"):
        fro = _weight_grad_check(name, got[name], ref[name])
        print(f"layer backward {case} {name}: rel {fro:.3e}")
