"""Plain, slow, fp64 CPU oracle of the LatentMoE layer's backward pass and of
the NVFP4 training recipe's pieces.

TEST INFRASTRUCTURE. Only the test suite may import this module. The CUDA
library never calls it and shares no code with it.

What it computes.

* ``backward``: the gradients of the layer forward of ``lmoe_oracle`` (its
  fp64 form, no rounding points) with respect to x and every weight, for an
  upstream gradient dout [T, d]. The layer is the one of the Nemotron 3
  whitepaper as summarised on the greeksharifa page, section 2.2 "LatentMoE"
  (router and shared experts on the d-dim x, routed experts in the latent l).
  The choice of the K experts is piecewise constant in the logits, so away
  from ties the router receives gradient only through the K renormalised
  gates g_k = exp(l_k) / sum_j exp(l_j) (j over the chosen K), whose
  derivative is dg_k / dl_j = g_k (delta_kj - g_j) for chosen j and 0 for the
  others.
* The NVFP4 training recipe named on the same page, section 2.4 "NVFP4
  Training", and on the Japanese summary page, section 4 "NVFP4 pre-training":
  weights, activations and gradients are quantised so that fprop, dgrad and
  wgrad run as NVFP4 GEMMs; weights use two-dimensional scale blocks; the
  inputs of wgrad get a random Hadamard transform; gradients are rounded
  stochastically. The pages give no more detail; the readings taken:
  - RHT: 16-point blocks along the contraction dimension, each block v mapped
    to H16 diag(s) v / 4 with H16 the Sylvester Hadamard matrix and s a
    random +-1 vector of 16 signs shared by all blocks (an input). It is
    orthonormal, so it leaves an unquantised wgrad product unchanged.
  - Stochastic rounding of an element to E2M1: between its two grid
    neighbours lo <= |v| < hi it takes hi when u * (hi - lo) < |v| - lo for a
    uniform u in [0, 1) (an input, one per element), else lo; |v| >= 6
    saturates to 6; the sign is kept. The block scales still round to
    nearest even.
  - Which operand gets what, for one linear layer Y = X W^T: dgrad
    dX = dY W quantises dY along its rows (the contraction dim) with
    stochastic rounding and W with 16 x 16 blocks (the fprop codes, as 2-D
    blocks quantise W and W^T alike); wgrad dW = dY^T X transforms dY and X
    along the tokens (the contraction dim), then quantises both along the
    tokens, dY with stochastic rounding and X to nearest.
  - The uniforms: passed in, or drawn by ``sr_uniforms`` from Philox-4x32-10
    (the counter-based generator of Salmon et al., SC11), which a kernel can
    evaluate element by element from the same published definition.
* ``backward_nvfp4``: the layer's gradients with only its routed experts'
  GEMMs under that recipe (NVFP4 z, a and 2-D-block weights in their
  forward; ``nvfp4_linear_backward`` for their dgrad and wgrad, each
  expert's rows padded with zero rows to a multiple of 16); the router, the
  latent projections and the shared experts stay unquantised, and every
  quantiser passes its gradient straight through.
"""
from __future__ import annotations

import numpy as np

from . import lmoe_oracle as O

# ----------------------------------------------------------------------------
# The layer's gradients (fp64)
# ----------------------------------------------------------------------------


class ParamWeights:
    """fp64 weights in the interface ``lmoe_oracle.forward`` reads
    (``dense(key)``, ``expert(key, e)``, storage tag ``st``)."""

    def __init__(self, params: dict):
        self.p = params
        self.st = "f64"

    def dense(self, key):
        return self.p[key]

    def expert(self, key, e):
        return self.p[key][e]


def params_from_inputs(wl, inp) -> dict:
    """fp64 values of a workload's stored inputs, as the layer reads them
    (NVFP4 expert matrices dequantised)."""
    W = O._Weights(wl, inp)
    p = {"x": W.dense("x"), "w_router": W.dense("w_router"), "router_bias": inp.get("router_bias")}
    p["w_down"] = None if wl.identity else W.dense("w_down")
    p["w_up"] = None if wl.identity else W.dense("w_up")
    p["w1"] = np.stack([W.expert("w1", e) for e in range(wl.N)])
    p["w2"] = np.stack([W.expert("w2", e) for e in range(wl.N)])
    p["ws1"] = W.dense("ws1") if wl.n_shared else None
    p["ws2"] = W.dense("ws2") if wl.n_shared else None
    return p


def backward(params: dict, K: int, dout) -> dict:
    """Gradients of out = layer(params) contracted with dout [T, d].

    params: fp64 arrays x [T, d], w_router [N, d], router_bias [N] or None,
    w_down [l, d] / w_up [d, l] (both None for identity projections),
    w1 [N, m, l], w2 [N, l, m], ws1 [S, m_s, d] / ws2 [S, d, m_s] or None.

    Returns dx, dw_router, drouter_bias (None without a bias), dw_down,
    dw_up (None for identity), dw1, dw2, dws1, dws2 (None without shared
    experts), and the forward's idx and gates.
    """
    x = np.asarray(params["x"], dtype=np.float64)
    dout = np.asarray(dout, dtype=np.float64)
    T = x.shape[0]
    wr, bias = params["w_router"], params.get("router_bias")
    w_down, w_up = params.get("w_down"), params.get("w_up")
    w1, w2 = params["w1"], params["w2"]
    N = w1.shape[0]

    # forward quantities the gradients need
    logits = O.router_logits(x, wr, bias)
    idx, gates = O.route_topk(logits, K)
    z = x if w_down is None else x @ w_down.T

    # up-projection: out = c W_up^T (+ shared); c = sum_k g_k o_k
    dc = dout if w_up is None else dout @ w_up
    c = np.zeros((T, z.shape[1]))
    dz = np.zeros_like(z)
    dgate = np.zeros((T, K))
    dw1 = np.zeros_like(w1)
    dw2 = np.zeros_like(w2)
    for e in range(N):
        t, k = np.nonzero(idx == e)          # the slots routed to expert e
        if t.size == 0:
            continue
        ze = z[t]
        h = ze @ w1[e].T                     # [n_e, m]
        a = O.sq_relu(h)
        o = a @ w2[e].T                      # ungated expert output [n_e, l]
        g = gates[t, k]
        np.add.at(c, t, g[:, None] * o)
        dy = dc[t]                           # gradient reaching each slot's gated output
        dgate[t, k] = np.sum(dy * o, axis=1)
        do = g[:, None] * dy
        dw2[e] = do.T @ a
        dh = (do @ w2[e]) * 2.0 * np.maximum(h, 0.0)
        dw1[e] = dh.T @ ze
        np.add.at(dz, t, dh @ w1[e])
    dw_up = None if w_up is None else dout.T @ c

    # gates -> logits (renormalised softmax over the chosen K)
    dsel = gates * (dgate - np.sum(gates * dgate, axis=1, keepdims=True))
    dlogits = np.zeros((T, N))
    np.put_along_axis(dlogits, idx.astype(np.int64), dsel, axis=1)
    dw_router = dlogits.T @ x
    dbias = None if bias is None else np.sum(dlogits, axis=0)
    dx = dlogits @ wr

    # down-projection
    if w_down is None:
        dw_down = None
        dx = dx + dz
    else:
        dw_down = dz.T @ x
        dx = dx + dz @ w_down

    # shared experts on x: out += relu(x Ws1_s^T)^2 Ws2_s^T
    dws1 = dws2 = None
    if params.get("ws1") is not None:
        ws1, ws2 = params["ws1"], params["ws2"]
        dws1, dws2 = np.zeros_like(ws1), np.zeros_like(ws2)
        for s in range(ws1.shape[0]):
            pre = x @ ws1[s].T
            hs = O.sq_relu(pre)
            dws2[s] = dout.T @ hs
            dpre = (dout @ ws2[s]) * 2.0 * np.maximum(pre, 0.0)
            dws1[s] = dpre.T @ x
            dx = dx + dpre @ ws1[s]

    return dict(dx=dx, dw_router=dw_router, drouter_bias=dbias, dw_down=dw_down, dw_up=dw_up,
                dw1=dw1, dw2=dw2, dws1=dws1, dws2=dws2, idx=idx, gates=gates)


# ----------------------------------------------------------------------------
# NVFP4 training pieces
# ----------------------------------------------------------------------------


def hadamard16() -> np.ndarray:
    """The 16 x 16 Sylvester Hadamard matrix (entries +-1): H_1 = [1],
    H_2n = [[H_n, H_n], [H_n, -H_n]]."""
    H = np.ones((1, 1))
    while H.shape[0] < 16:
        H = np.block([[H, H], [H, -H]])
    return H


def rht(X, signs, axis: int = 0) -> np.ndarray:
    """Random Hadamard transform of X along ``axis`` (its length a multiple of
    16): every block of 16 consecutive entries v becomes H16 diag(signs) v / 4."""
    X = np.asarray(X, dtype=np.float64)
    signs = np.asarray(signs, dtype=np.float64)
    assert signs.shape == (16,) and np.all(np.abs(signs) == 1.0)
    Xm = np.moveaxis(X, axis, 0)
    n = Xm.shape[0]
    assert n % 16 == 0
    M = hadamard16() * signs[None, :] / 4.0
    blocks = Xm.reshape((n // 16, 16) + Xm.shape[1:])
    out = np.einsum("ij,bj...->bi...", M, blocks).reshape(Xm.shape)
    return np.moveaxis(out, 0, axis)


def e2m1_sr_encode(v, u) -> np.ndarray:
    """Stochastic rounding to E2M1 codes: |v| >= 6 -> 6; otherwise, with
    lo <= |v| < hi the neighbouring grid points, hi if u * (hi - lo) < |v| - lo
    else lo (exact comparison; u in [0, 1)). The sign bit is the sign of v."""
    v = np.asarray(v, dtype=np.float64)
    u = np.broadcast_to(np.asarray(u, dtype=np.float64), v.shape)
    a = np.abs(v)
    grid = O.E2M1_MAG
    lo_i = np.clip(np.searchsorted(grid, a, side="right") - 1, 0, len(grid) - 1)
    hi_i = np.minimum(lo_i + 1, len(grid) - 1)
    lo, hi = grid[lo_i], grid[hi_i]
    up = (hi_i > lo_i) & (u * (hi - lo) < a - lo)
    code = np.where(a >= O.E2M1_MAX, len(grid) - 1, np.where(up, hi_i, lo_i))
    return (code | np.where(np.signbit(v), 8, 0)).astype(np.uint8)


def nvfp4_quantize_sr(X, u, s_g: float | None = None):
    """``lmoe_oracle.nvfp4_quantize`` with the element step rounded
    stochastically (u [rows, cols] uniforms in [0, 1)); the global and block
    scales are the round-to-nearest ones of that function."""
    X = np.asarray(X, dtype=np.float64)
    rows, cols = X.shape
    _, sb_code, s_g = O.nvfp4_quantize(X, s_g)
    sb = O.e4m3_decode(sb_code)
    sc = O.round_f32(sb * s_g)
    blocks = X.reshape(rows, cols // O.NVFP4_BLOCK, O.NVFP4_BLOCK)
    with np.errstate(divide="ignore", invalid="ignore"):
        v = O.round_f32(blocks / sc[..., None])
    q = e2m1_sr_encode(v, np.asarray(u, dtype=np.float64).reshape(blocks.shape))
    q = np.where((sb == 0.0)[..., None], np.uint8(0), q).astype(np.uint8).reshape(rows, cols)
    codes = (q[:, 0::2] | (q[:, 1::2] << 4)).astype(np.uint8)
    return codes, sb_code, s_g


# Philox-4x32-10 (Salmon et al., "Parallel random numbers: as easy as 1, 2, 3",
# SC11, section 5): the counter-based generator both sides of a stochastic
# rounding kernel can evaluate independently, element by element.
_PHILOX_M = (0xD2511F53, 0xCD9E8D57)
_PHILOX_W = (0x9E3779B9, 0xBB67AE85)


def philox4x32_10(counter, key) -> np.ndarray:
    """Philox-4x32-10 of counters [..., 4] (uint32 words) under key [2]:
    ten rounds; each round takes the 64-bit products of words 0 and 2 with the
    two multipliers and sets (hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0); the key
    grows by the two Weyl constants between rounds. Returns [..., 4] uint32."""
    c = np.asarray(counter, dtype=np.uint64) & np.uint64(0xFFFFFFFF)
    k0, k1 = (int(v) & 0xFFFFFFFF for v in key)
    c0, c1, c2, c3 = (c[..., i] for i in range(4))
    m32 = np.uint64(0xFFFFFFFF)
    for r in range(10):
        if r:
            k0 = (k0 + _PHILOX_W[0]) & 0xFFFFFFFF
            k1 = (k1 + _PHILOX_W[1]) & 0xFFFFFFFF
        p0 = c0 * np.uint64(_PHILOX_M[0])
        p1 = c2 * np.uint64(_PHILOX_M[1])
        c0, c1, c2, c3 = ((p1 >> np.uint64(32)) ^ c1 ^ np.uint64(k0), p1 & m32,
                          (p0 >> np.uint64(32)) ^ c3 ^ np.uint64(k1), p0 & m32)
    return np.stack([c0, c1, c2, c3], axis=-1).astype(np.uint32)


def sr_uniforms(n: int, seed: int, stream: int = 0) -> np.ndarray:
    """n uniforms in [0, 1) for stochastic rounding, element i from word i % 4
    of Philox-4x32-10 at counter (i // 4 low word, i // 4 high word, stream, 0)
    under key (seed low word, seed high word): u = (word >> 8) * 2^-24, a
    24-bit value every fp32 holds exactly."""
    i = np.arange((n + 3) // 4, dtype=np.uint64)
    ctr = np.stack([i & np.uint64(0xFFFFFFFF), i >> np.uint64(32),
                    np.full_like(i, stream & 0xFFFFFFFF), np.zeros_like(i)], axis=-1)
    words = philox4x32_10(ctr, (seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF)).reshape(-1)[:n]
    return (words >> np.uint32(8)).astype(np.float64) * 2.0 ** -24


def _deq(q):
    return O.nvfp4_dequantize(*q)


def nvfp4_linear_backward(X, W, dY, signs, u_dgrad, u_wgrad, quantize: bool = True) -> dict:
    """dgrad and wgrad of one linear layer Y = X W^T under the NVFP4 training
    recipe (readings in the module docstring); products summed in fp64.

    X [T, n_in], W [n_out, n_in], dY [T, n_out] (T, n_in, n_out multiples of
    16); signs [16]; u_dgrad [T, n_out] and u_wgrad [n_out, T] uniforms.
    quantize=False makes every quantiser the identity (the transform stays),
    which leaves the plain products dY W and dY^T X.
    Returns dX [T, n_in] and dW [n_out, n_in].
    """
    X, W, dY = (np.asarray(a, dtype=np.float64) for a in (X, W, dY))
    q_sr = (lambda A, u: _deq(nvfp4_quantize_sr(A, u))) if quantize else (lambda A, u: A)
    q_2d = (lambda A: _deq(O.nvfp4_quantize_2d(A))) if quantize else (lambda A: A)
    q_rn = (lambda A: _deq(O.nvfp4_quantize(A))) if quantize else (lambda A: A)
    # dgrad: contraction over n_out; dY along its rows, W with 2-D blocks
    dX = q_sr(dY, u_dgrad) @ q_2d(W)
    # wgrad: contraction over the tokens; both operands transformed and
    # quantised along the tokens
    dYt = rht(dY, signs, axis=0).T          # [n_out, T]
    Xt = rht(X, signs, axis=0).T            # [n_in, T]
    dW = q_sr(dYt, u_wgrad) @ q_rn(Xt).T
    return dict(dX=dX, dW=dW)


def _fake_quant(A, s_g=None):
    return O.nvfp4_fake_quant(A, s_g)[0]


def routed_experts_backward_nvfp4(zq, w1, w2, idx, gates, dc, signs, seed: int, a_global_scale=None,
                                  quantize: bool = True) -> dict:
    """The routed experts' part of ``backward_nvfp4``, per expert e over the
    slots routed to it (t, k with idx[t, k] == e, in token order):

      forward (recomputed): h = ze W1q^T, aq = NVFP4(relu(h)^2, a_global_scale
        or the current amax), o = aq W2q^T, with ze = zq[t] (the NVFP4 latent
        rows) and W1q, W2q the experts' matrices quantised with 16 x 16 blocks;
      dgate[t, k] = dy . o with dy = dc[t];  do = gate * dy;
      dgrad and wgrad of the two GEMMs by ``nvfp4_linear_backward``, each
        expert's rows padded by zero rows to a multiple of 16, uniforms from
        ``sr_uniforms(seed, 4 e + 2 g + j)`` (g: 0 first GEMM, 1 second; j: 0
        dgrad, 1 wgrad);  dh = dA * 2 max(h, 0).

    Returns c [T, l] (the gated sum of the experts' outputs), dz [T, l] (the
    gradient reaching zq), dgate [T, K], dw1 [N, m, l] and dw2 [N, l, m].
    quantize=False turns every quantiser into the identity.
    """
    zq, dc, gates = (np.asarray(a, dtype=np.float64) for a in (zq, dc, gates))
    w1, w2 = np.asarray(w1, dtype=np.float64), np.asarray(w2, dtype=np.float64)
    T, l = zq.shape
    K = idx.shape[1]
    N = w1.shape[0]
    fq = _fake_quant if quantize else (lambda A, s_g=None: A)
    fq2 = (lambda A: _deq(O.nvfp4_quantize_2d(A))) if quantize else (lambda A: A)
    c = np.zeros((T, l))
    dz = np.zeros((T, l))
    dgate = np.zeros((T, K))
    dw1, dw2 = np.zeros_like(w1), np.zeros_like(w2)

    def pad16(A):
        R = -(-A.shape[0] // 16) * 16
        out = np.zeros((R,) + A.shape[1:])
        out[:A.shape[0]] = A
        return out

    def uni(rows, cols, stream):
        return sr_uniforms(rows * cols, seed, stream).reshape(rows, cols)

    for e in range(N):
        t, k = np.nonzero(idx == e)
        n = t.size
        if n == 0:
            continue
        ze = zq[t]
        h = ze @ fq2(w1[e]).T
        aq = fq(O.sq_relu(h), a_global_scale)
        o = aq @ fq2(w2[e]).T
        g = gates[t, k]
        np.add.at(c, t, g[:, None] * o)
        dy = dc[t]
        dgate[t, k] = np.sum(dy * o, axis=1)
        do = g[:, None] * dy
        R = -(-n // 16) * 16
        r2 = nvfp4_linear_backward(pad16(aq), w2[e], pad16(do), signs, uni(R, l, 4 * e + 2),
                                   uni(l, R, 4 * e + 3), quantize)
        dw2[e] = r2["dW"]
        dh = r2["dX"][:n] * 2.0 * np.maximum(h, 0.0)
        r1 = nvfp4_linear_backward(pad16(ze), w1[e], pad16(dh), signs, uni(R, w1.shape[1], 4 * e + 0),
                                   uni(w1.shape[1], R, 4 * e + 1), quantize)
        dw1[e] = r1["dW"]
        np.add.at(dz, t, r1["dX"][:n])
    return dict(c=c, dz=dz, dgate=dgate, dw1=dw1, dw2=dw2)


def backward_nvfp4(params: dict, K: int, dout, signs, seed: int, a_global_scale=None,
                   quantize: bool = True) -> dict:
    """The layer's gradients with its routed experts trained under the NVFP4
    recipe: the expert GEMMs' forward reads NVFP4 z (of z rounded to BF16, the
    forward's rounding point; current amax), NVFP4 a
    (``a_global_scale``, else its current amax) and 2-D-block NVFP4 weights;
    their dgrad and wgrad are ``nvfp4_linear_backward``, with each expert's
    rows padded by zero rows to a multiple of 16 for the token transform. The
    router, the latent projections and the shared experts stay unquantised
    (the recipe keeps such layers in higher precision; the latent projections
    stay BF16 on the pages), and every quantiser passes its gradient straight
    through. Uniforms come from ``sr_uniforms(seed, stream)`` with stream
    4 e + 2 g + j for expert e, GEMM g (0: first, 1: second) and j (0: dgrad,
    1: wgrad). quantize=False turns every quantiser into the identity.
    Returns the same keys as ``backward``.
    """
    x = np.asarray(params["x"], dtype=np.float64)
    dout = np.asarray(dout, dtype=np.float64)
    T = x.shape[0]
    wr, bias = params["w_router"], params.get("router_bias")
    w_down, w_up = params.get("w_down"), params.get("w_up")
    w1, w2 = params["w1"], params["w2"]
    N = w1.shape[0]
    fq = _fake_quant if quantize else (lambda A, s_g=None: A)

    logits = O.router_logits(x, wr, bias)
    idx, gates = O.route_topk(logits, K)
    z = x if w_down is None else x @ w_down.T
    # the experts read NVFP4 of z as the forward stores it: rounded to BF16
    # first (its rounding point), then quantised with the current amax
    zq = fq(O.round_bf16(z)) if quantize else z
    dc = dout if w_up is None else dout @ w_up
    r = routed_experts_backward_nvfp4(zq, w1, w2, idx, gates, dc, signs, seed, a_global_scale, quantize)
    c, dz, dgate, dw1, dw2 = r["c"], r["dz"], r["dgate"], r["dw1"], r["dw2"]
    dw_up = None if w_up is None else dout.T @ c

    dsel = gates * (dgate - np.sum(gates * dgate, axis=1, keepdims=True))
    dlogits = np.zeros((T, N))
    np.put_along_axis(dlogits, idx.astype(np.int64), dsel, axis=1)
    dw_router = dlogits.T @ x
    dbias = None if bias is None else np.sum(dlogits, axis=0)
    dx = dlogits @ wr
    if w_down is None:
        dw_down = None
        dx = dx + dz
    else:
        dw_down = dz.T @ x
        dx = dx + dz @ w_down
    dws1 = dws2 = None
    if params.get("ws1") is not None:
        ws1, ws2 = params["ws1"], params["ws2"]
        dws1, dws2 = np.zeros_like(ws1), np.zeros_like(ws2)
        for s in range(ws1.shape[0]):
            pre = x @ ws1[s].T
            dws2[s] = dout.T @ O.sq_relu(pre)
            dpre = (dout @ ws2[s]) * 2.0 * np.maximum(pre, 0.0)
            dws1[s] = dpre.T @ x
            dx = dx + dpre @ ws1[s]
    return dict(dx=dx, dw_router=dw_router, drouter_bias=dbias, dw_down=dw_down, dw_up=dw_up,
                dw1=dw1, dw2=dw2, dws1=dws1, dws2=dws2, idx=idx, gates=gates)
