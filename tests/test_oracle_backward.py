"""Pins of the backward-pass oracle (CPU), each independent of the code it checks:

* the layer gradients against central finite differences of the forward
  oracle (itself pinned in test_oracle_forward.py), and against torch
  autograd through a dense forward written here (every expert applied to
  every token, gates from a masked softmax) -- a different computation;
* special cases: K = 1 leaves the router without gradient; linearity in dout;
* the NVFP4 training pieces against closed forms: the Sylvester Hadamard
  entries (-1)^popcount(i & j), orthonormality of the transform, the exact
  mean of stochastic rounding over a uniform grid of u, and exact dgrad /
  wgrad products on operands constructed to be exactly representable.
"""
import numpy as np
import pytest
import torch

import lmoe_inputs as LI
from oracle import lmoe_backward as B
from oracle import lmoe_oracle as O

GRADS = ("dx", "dw_router", "drouter_bias", "dw_down", "dw_up", "dw1", "dw2", "dws1", "dws2")
PARAM_OF = {"dx": "x", "dw_router": "w_router", "drouter_bias": "router_bias", "dw_down": "w_down",
            "dw_up": "w_up", "dw1": "w1", "dw2": "w2", "dws1": "ws1", "dws2": "ws2"}


def _params(seed, T=6, d=16, l=8, N=6, m=8, S=1, ms=8, identity=False, bias=True):
    rng = np.random.default_rng(seed)
    if identity:
        l = d
    n = rng.standard_normal
    return dict(
        x=n((T, d)), w_router=n((N, d)) / np.sqrt(d), router_bias=n(N) if bias else None,
        w_down=None if identity else n((l, d)) / np.sqrt(d), w_up=None if identity else n((d, l)) / np.sqrt(l),
        w1=n((N, m, l)) / np.sqrt(l), w2=n((N, l, m)) / np.sqrt(m),
        ws1=n((S, ms, d)) / np.sqrt(d) if S else None, ws2=n((S, d, ms)) / np.sqrt(ms) if S else None)


def _workload(p, K):
    T, d = p["x"].shape
    N, m, l = p["w1"].shape
    S = 0 if p["ws1"] is None else p["ws1"].shape[0]
    ms = 0 if p["ws1"] is None else p["ws1"].shape[1]
    return LI.Workload("bwd", T=T, d=d, l=l, N=N, K=K, m=m, n_shared=S, m_shared=ms, identity=p["w_down"] is None)


def _out(p, K):
    """The forward oracle's unrounded output for fp64 parameters."""
    inp = {"x": p["x"], "router_bias": p["router_bias"], "ws1": p["ws1"], "ws2": p["ws2"]}
    return O.forward(_workload(p, K), inp, precision="f64", weights=B.ParamWeights(p))["out_unrounded"]


def _min_gap(p, K):
    lg = O.router_logits(p["x"], p["w_router"], p["router_bias"])
    s = -np.sort(-lg, axis=1)
    return float(np.min(s[:, K - 1] - s[:, K]))


@pytest.mark.parametrize("identity,S,bias", [(False, 1, True), (True, 2, False), (False, 0, True)])
def test_gradients_match_central_differences_of_the_forward_oracle(identity, S, bias):
    K = 2
    p = _params(11 + S, identity=identity, S=S, bias=bias)
    assert _min_gap(p, K) > 1e-3          # the chosen experts stay put under the steps
    rng = np.random.default_rng(3)
    dout = rng.standard_normal((p["x"].shape[0], p["x"].shape[1]))
    g = B.backward(p, K, dout)
    h = 1e-5
    for gname in GRADS:
        pname = PARAM_OF[gname]
        if p[pname] is None:
            assert g[gname] is None
            continue
        flat = p[pname].reshape(-1)
        picks = rng.choice(flat.size, size=min(flat.size, 10), replace=False)
        for i in picks:
            keep = flat[i]
            flat[i] = keep + h
            up = np.sum(dout * _out(p, K))
            flat[i] = keep - h
            dn = np.sum(dout * _out(p, K))
            flat[i] = keep
            fd = (up - dn) / (2 * h)
            an = g[gname].reshape(-1)[i]
            assert abs(fd - an) <= 1e-6 * (1.0 + abs(an)), (gname, i, fd, an)


def _torch_dense_forward(P, idx):
    """Dense formulation: out = sum_e G[:, e] * FFN_e(z) projected up, plus the
    shared experts; G = softmax of the logits restricted to the chosen experts."""
    x = P["x"]
    logits = x @ P["w_router"].T
    if P["router_bias"] is not None:
        logits = logits + P["router_bias"]
    T, N = logits.shape
    mask = torch.zeros((T, N), dtype=torch.bool)
    mask[torch.arange(T)[:, None], torch.as_tensor(idx, dtype=torch.long)] = True
    G = torch.softmax(logits.masked_fill(~mask, float("-inf")), dim=1)
    z = x if P["w_down"] is None else x @ P["w_down"].T
    y = 0.0
    for e in range(N):
        y = y + G[:, e:e + 1] * (torch.relu(z @ P["w1"][e].T) ** 2 @ P["w2"][e].T)
    out = y if P["w_up"] is None else y @ P["w_up"].T
    if P["ws1"] is not None:
        for s in range(P["ws1"].shape[0]):
            out = out + torch.relu(x @ P["ws1"][s].T) ** 2 @ P["ws2"][s].T
    return out


@pytest.mark.parametrize("identity,S,K", [(False, 2, 3), (True, 1, 2), (False, 0, 1), (False, 1, 6)])
def test_gradients_match_autograd_of_a_dense_forward(identity, S, K):
    p = _params(29 + K, T=9, identity=identity, S=S)
    rng = np.random.default_rng(4)
    dout = rng.standard_normal((9, p["x"].shape[1]))
    g = B.backward(p, K, dout)
    P = {k: (None if v is None else torch.tensor(v, dtype=torch.float64, requires_grad=True)) for k, v in p.items()}
    out = _torch_dense_forward(P, g["idx"])
    assert np.allclose(out.detach().numpy(), _out(p, K), rtol=1e-12, atol=1e-12)
    (out * torch.tensor(dout)).sum().backward()
    for gname in GRADS:
        t = P[PARAM_OF[gname]]
        if t is None:
            assert g[gname] is None
            continue
        assert np.allclose(g[gname], t.grad.numpy(), rtol=1e-10, atol=1e-12), gname


def test_top_1_routing_gives_the_router_no_gradient():
    p = _params(5, N=5)
    g = B.backward(p, 1, np.random.default_rng(1).standard_normal((6, 16)))
    assert np.all(g["dw_router"] == 0.0) and np.all(g["drouter_bias"] == 0.0)
    assert np.all(g["gates"] == 1.0)


def test_gradients_are_linear_in_dout():
    p = _params(8)
    rng = np.random.default_rng(2)
    a, b = rng.standard_normal((6, 16)), rng.standard_normal((6, 16))
    ga, gb, gab = B.backward(p, 2, a), B.backward(p, 2, b), B.backward(p, 2, a - 3.0 * b)
    for k in GRADS:
        assert np.allclose(gab[k], ga[k] - 3.0 * gb[k], rtol=1e-12, atol=1e-12), k


def test_params_from_inputs_reads_the_stored_values():
    wl = LI.reduced("ultra_decode", T=4, d=64, l=32, N=8, K=2, m=32)
    inp = LI.make_inputs(wl)
    p = B.params_from_inputs(wl, inp)
    assert np.array_equal(p["x"], O.from_bf16_bits(inp["x"]))
    assert np.array_equal(p["w1"][3], O.from_bf16_bits(inp["w1"][3]))
    assert np.allclose(_out(p, wl.K), O.forward(wl, inp, precision="f64")["out_unrounded"], rtol=0, atol=0)


# ----------------------------------------------------------------------------
# NVFP4 training pieces
# ----------------------------------------------------------------------------


def test_hadamard16_entries_and_orthogonality():
    H = B.hadamard16()
    i, j = np.meshgrid(np.arange(16), np.arange(16), indexing="ij")
    popc = np.vectorize(lambda v: bin(v).count("1"))(i & j)
    assert np.array_equal(H, (-1.0) ** popc)
    assert np.array_equal(H @ H.T, 16.0 * np.eye(16))


def test_rht_is_orthonormal_blockwise_and_keeps_products():
    rng = np.random.default_rng(7)
    s = rng.choice([-1.0, 1.0], 16)
    A, C = rng.standard_normal((48, 5)), rng.standard_normal((48, 7))
    RA, RC = B.rht(A, s, axis=0), B.rht(C, s, axis=0)
    assert np.allclose(RA.T @ RC, A.T @ C, rtol=1e-12, atol=1e-12)       # an unquantised wgrad is unchanged
    assert np.allclose(np.linalg.norm(RA, axis=0), np.linalg.norm(A, axis=0), rtol=1e-13)
    # inverse: diag(s) H / 4 per block
    back = np.concatenate([(s[:, None] * (B.hadamard16() @ RA[b:b + 16])) / 4.0 for b in range(0, 48, 16)])
    assert np.allclose(back, A, rtol=1e-13, atol=1e-13)
    # blocks do not mix: a change in block 1 leaves blocks 0 and 2 alone
    A2 = A.copy()
    A2[20, 3] += 1.0
    d = B.rht(A2, s, axis=0) - RA
    assert np.all(d[:16] == 0.0) and np.all(d[32:] == 0.0) and np.any(d[16:32] != 0.0)
    # along another axis: the transpose of the same transform
    assert np.allclose(B.rht(A.T, s, axis=1), RA.T, rtol=0, atol=0)


def test_stochastic_rounding_grid_values_and_neighbours():
    u = np.linspace(0.0, 1.0, 97, endpoint=False)
    for mag, code in zip(O.E2M1_MAG, range(8)):
        for sign in (1.0, -1.0):
            got = B.e2m1_sr_encode(np.full(u.shape, sign * mag), u)
            assert np.all(got == (code | (8 if sign < 0 else 0)))
    rng = np.random.default_rng(9)
    v = rng.uniform(-7.0, 7.0, 5000)
    q = O.e2m1_decode(B.e2m1_sr_encode(v, rng.random(5000)))
    a = np.minimum(np.abs(v), 6.0)
    lo = O.E2M1_MAG[np.searchsorted(O.E2M1_MAG, a, side="right") - 1]
    hi = O.E2M1_MAG[np.minimum(np.searchsorted(O.E2M1_MAG, a, side="right"), 7)]
    assert np.all((np.abs(q) == lo) | (np.abs(q) == hi))
    assert np.all(np.sign(q)[q != 0] == np.sign(v)[q != 0])
    assert np.all(np.abs(q[np.abs(v) >= 6.0]) == 6.0)                   # saturation


def test_stochastic_rounding_mean_over_a_uniform_grid_is_exact():
    """With u_i = i / M, the value rounds up for i < p M (p = (|v| - lo) / (hi - lo)),
    so for p M an integer the mean of the rounded values is v exactly."""
    M = 1024
    u = np.arange(M) / M
    for lo, hi in zip(O.E2M1_MAG[:-1], O.E2M1_MAG[1:]):
        for j in (1, 37, 512, 1023):
            v = lo + (hi - lo) * j / M
            for sign in (1.0, -1.0):
                q = O.e2m1_decode(B.e2m1_sr_encode(np.full(M, sign * v), u))
                assert np.sum(q) / M == sign * v
    # u = 0 rounds every off-grid magnitude up; the largest u below 1 rounds it down
    assert O.e2m1_decode(B.e2m1_sr_encode(np.array([1.1]), 0.0))[0] == 1.5
    assert O.e2m1_decode(B.e2m1_sr_encode(np.array([1.1]), 1.0 - 2.0 ** -24))[0] == 1.0


def _exact_rows(rng, rows, cols):
    """1 x 16 blocks of grid points times a power-of-two (or 448) block scale,
    one +-6 per block, one block at 448: with the current amax s_g = 1 and
    every fp32 step of the quantiser exact."""
    X = np.zeros((rows, cols))
    for r in range(rows):
        for b in range(cols // 16):
            sb = 448.0 if (r, b) == (0, 0) else 2.0 ** rng.integers(-6, 8)
            q = rng.choice(O.E2M1_MAG, 16) * rng.choice([-1.0, 1.0], 16)
            q[rng.integers(16)] = 6.0 * rng.choice([-1.0, 1.0])
            X[r, b * 16:(b + 1) * 16] = q * sb
    return X


def _exact_2d(rng, rows, cols):
    X = np.zeros((rows, cols))
    for rb in range(rows // 16):
        for cb in range(cols // 16):
            sb = 448.0 if (rb, cb) == (0, 0) else 2.0 ** rng.integers(-5, 7)
            q = rng.choice(O.E2M1_MAG, (16, 16)) * rng.choice([-1.0, 1.0], (16, 16))
            q[rng.integers(16), rng.integers(16)] = 6.0
            X[rb * 16:(rb + 1) * 16, cb * 16:(cb + 1) * 16] = q * sb
    return X


def test_sr_quantiser_keeps_the_scales_and_is_exact_on_representable_input():
    rng = np.random.default_rng(12)
    X = _exact_rows(rng, 4, 64)
    c, sf, g = B.nvfp4_quantize_sr(X, rng.random(X.shape))
    c0, sf0, g0 = O.nvfp4_quantize(X)
    assert g == g0 == 1.0 and np.array_equal(sf, sf0)
    assert np.array_equal(O.nvfp4_dequantize(c, sf, g), X)          # grid points never move


def test_sr_quantiser_is_unbiased_over_a_uniform_grid():
    """A block with its scale pinned by a +-6 entry (s_b = 1, s_g = 1) and the
    other entries at k/64 of the way between grid neighbours: the mean over
    u_i = i/64 of the dequantised values is the input exactly."""
    M = 64
    X = np.zeros((1, 16))
    X[0, 0] = 6.0
    vals = [0.5 + 0.5 * 3 / M, 1.0 + 0.5 * 17 / M, 2.0 + 1.0 * 40 / M, 4.0 + 2.0 * 63 / M, -(3.0 + 1.0 * 5 / M)]
    X[0, 1:1 + len(vals)] = vals
    acc = np.zeros_like(X)
    for i in range(M):
        c, sf, g = B.nvfp4_quantize_sr(X, np.full(X.shape, i / M), s_g=1.0)
        assert O.e4m3_decode(sf)[0, 0] == 1.0
        acc += O.nvfp4_dequantize(c, sf, g)
    assert np.array_equal(acc / M, X)


def test_nvfp4_dgrad_exact_on_representable_operands():
    rng = np.random.default_rng(14)
    T, n_in, n_out = 32, 48, 32
    dY = _exact_rows(rng, T, n_out)          # blocks along n_out: dgrad's contraction dim
    W = _exact_2d(rng, n_out, n_in)
    X = rng.standard_normal((T, n_in))
    s = rng.choice([-1.0, 1.0], 16)
    r = B.nvfp4_linear_backward(X, W, dY, s, rng.random((T, n_out)), rng.random((n_out, T)))
    assert np.array_equal(r["dX"], dY @ W)


def test_nvfp4_wgrad_exact_when_the_transformed_operands_are_representable():
    """dY and X built as the inverse transform of exactly representable
    matrices (blocks along the tokens): the transform returns those matrices
    exactly, they quantise exactly, and dW equals dY^T X (to fp64 rounding of
    the reference product)."""
    rng = np.random.default_rng(15)
    T, n_in, n_out = 48, 32, 16
    s = rng.choice([-1.0, 1.0], 16)
    Hs = B.hadamard16()

    def inverse_rht(Y):
        return np.concatenate([(s[:, None] * (Hs @ Y[b:b + 16])) / 4.0 for b in range(0, Y.shape[0], 16)])

    Rd, Rx = _exact_rows(rng, n_out, T), _exact_rows(rng, n_in, T)
    dY, X = inverse_rht(Rd.T), inverse_rht(Rx.T)
    assert np.array_equal(B.rht(dY, s, axis=0), Rd.T) and np.array_equal(B.rht(X, s, axis=0), Rx.T)
    W = rng.standard_normal((n_out, n_in))
    r = B.nvfp4_linear_backward(X, W, dY, s, rng.random((T, n_out)), rng.random((n_out, T)))
    assert np.array_equal(r["dW"], Rd @ Rx.T)
    assert np.allclose(r["dW"], dY.T @ X, rtol=1e-12, atol=1e-9)


def test_philox_known_answer_vectors():
    rows = []
    with open(__file__.replace("test_oracle_backward.py", "golden/philox4x32_10_kat.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                rows.append([int(w, 16) for w in line.split()])
    assert len(rows) == 3
    for r in rows:
        got = B.philox4x32_10(np.array(r[:4], dtype=np.uint64), r[4:6])
        assert got.tolist() == r[6:10]
    # vectorised over counters: the same words as one call per counter
    ctrs = np.array([r[:4] for r in rows], dtype=np.uint64)
    assert B.philox4x32_10(ctrs, rows[0][4:6])[0].tolist() == rows[0][6:10]


def test_sr_uniforms_layout_and_range():
    u = B.sr_uniforms(10, seed=5, stream=2)
    w = B.philox4x32_10(np.array([[0, 0, 2, 0], [1, 0, 2, 0], [2, 0, 2, 0]], dtype=np.uint64), (5, 0)).reshape(-1)
    assert np.array_equal(u, (w[:10] >> 8).astype(np.float64) / 2.0 ** 24)
    big = B.sr_uniforms(1 << 20, seed=1)
    assert big.min() >= 0.0 and big.max() < 1.0
    assert np.all(big * 2.0 ** 24 == np.floor(big * 2.0 ** 24))         # 24-bit values
    assert abs(big.mean() - 0.5) < 5 * np.sqrt(1 / 12 / big.size)
    assert not np.array_equal(B.sr_uniforms(64, seed=1), B.sr_uniforms(64, seed=1, stream=1))


@pytest.mark.parametrize("identity,S", [(False, 1), (True, 0)])
def test_nvfp4_layer_backward_without_quantisation_is_the_exact_backward(identity, S):
    """With every quantiser the identity, the NVFP4 composition (per-expert
    padding, operand wiring, token transform) must reproduce the exact
    gradients: the transform is orthonormal and the padding rows are zero."""
    p = _params(41, T=21, d=32, l=32, N=5, m=48, S=S, ms=16, identity=identity)
    dout = np.random.default_rng(6).standard_normal((21, 32))
    s = np.random.default_rng(7).choice([-1.0, 1.0], 16)
    exact = B.backward(p, 2, dout)
    comp = B.backward_nvfp4(p, 2, dout, s, seed=3, quantize=False)
    for k in GRADS:
        if exact[k] is None:
            assert comp[k] is None
            continue
        assert np.allclose(comp[k], exact[k], rtol=1e-10, atol=1e-12), k


def test_nvfp4_layer_backward_seeds_and_quantisation():
    p = _params(43, T=40, d=32, l=32, N=4, m=32, S=0)
    dout = np.random.default_rng(8).standard_normal((40, 32))
    s = np.random.default_rng(9).choice([-1.0, 1.0], 16)
    a = B.backward_nvfp4(p, 2, dout, s, seed=1)
    b = B.backward_nvfp4(p, 2, dout, s, seed=1)
    c = B.backward_nvfp4(p, 2, dout, s, seed=2)
    for k in ("dx", "dw1", "dw2", "dw_router"):
        assert np.array_equal(a[k], b[k]), k                    # the uniforms are a function of the seed
    assert not np.array_equal(a["dw1"], c["dw1"])              # stochastic rounding depends on them
    exact = B.backward(p, 2, dout)
    for k in ("dx", "dw1", "dw2"):
        assert not np.allclose(a[k], exact[k], rtol=1e-6)      # the quantisers act
        cos = np.sum(a[k] * exact[k]) / (np.linalg.norm(a[k]) * np.linalg.norm(exact[k]))
        assert cos > 0.9, (k, cos)                              # and stay a gradient of the same layer
