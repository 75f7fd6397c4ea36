"""Plain, slow, fp64 CPU oracle of the LatentMoE layer forward.

TEST INFRASTRUCTURE. Only the test suite, the package's smoke check and the
benchmark's CPU-baseline leg may import this module. The CUDA library never
calls it and shares no code with it.

What it computes (Nemotron 3 whitepaper as summarised on the greeksharifa
page, section 2.2 "LatentMoE", and the notes.yuuk.io page, section 2
"LatentMoE"): each token's hidden state x in R^d is projected down to a latent
z in R^l (l < d), the routed experts run in l, their gate-weighted sum is
projected back to d. The router and the shared experts stay outside the
compression and read the d-dim x. NVFP4 (same greeksharifa page, section 2.4
"NVFP4 Training"): E2M1 elements, 16-element micro-blocks with an E4M3 scale,
and an FP32 per-tensor global scale.

Steps the pages leave open, with the reading taken (each is also a row of the
design notes):

* router score: softmax over all N experts; top-K by (logit descending, expert
  index ascending); the K gates renormalised to sum to one.
* expert FFN: squared ReLU, l -> m -> l; shared experts the same in d.
* permutation: a stable counting sort of the flat slots f = t*K + k by expert.
* NVFP4 scales: s_g = amax / (6 * 448) (1 when amax = 0); per 16-block
  s_b = E4M3(amax_b / (s_g * 6)); codes E2M1(x / (dec(s_b) * s_g)); both
  conversions round to nearest even and saturate to the largest finite value.
  Every step is an FP32 operation; it is emulated here as an fp64 operation
  followed by rounding to fp32, which is exact for +, -, *, / (53 >= 2*24 + 2).
* precision contract: the layer rounds at fixed points -- z, a, y, c, out (and
  the shared experts' hidden) -- to the workload's storage type (BF16 or
  fp32); under NVFP4, z and a are fake-quantised instead. Between those
  points this oracle carries fp64.

Parity pins: every function here is checked by ``tests/test_oracle_*.py``
against brute force on tiny inputs, closed-form format tables, a library
routine (torch's float8_e4m3fn / bfloat16 casts) or an invariant of the method.
"""
from __future__ import annotations

import itertools

import numpy as np

# ----------------------------------------------------------------------------
# Storage formats of the inputs
# ----------------------------------------------------------------------------


def from_bf16_bits(u: np.ndarray) -> np.ndarray:
    """BF16 bit patterns (uint16) -> exact float64 values."""
    u = np.asarray(u, dtype=np.uint16)
    return (u.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def to_f64(a, dtype: str) -> np.ndarray:
    """Stored tensor (uint16 BF16 bits, float32, or float64 values passed
    through with dtype "f64") -> exact float64 values."""
    if a is None:
        return None
    if dtype == "f64":
        return np.asarray(a, dtype=np.float64)
    if dtype == "f32":
        return np.asarray(a, dtype=np.float32).astype(np.float64)
    return from_bf16_bits(a)


# ----------------------------------------------------------------------------
# Rounding points
# ----------------------------------------------------------------------------


def round_to_precision(x: np.ndarray, mant_bits: int, min_exp: int) -> np.ndarray:
    """Round float64 values to nearest-even on a binary grid with ``mant_bits``
    fraction bits and smallest normal exponent ``min_exp`` (subnormals keep the
    quantum 2**(min_exp - mant_bits)). Overflow is not handled (not reached)."""
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)                       # x = f * 2**e, 0.5 <= |f| < 1
    e = np.maximum(e - 1, min_exp)           # exponent of the leading bit
    quantum = np.ldexp(1.0, e - mant_bits)
    return np.round(x / quantum) * quantum   # np.round is round-half-even; /quantum is exact


def round_bf16(x):
    """Round to the nearest BF16 value (ties to even)."""
    return round_to_precision(x, 7, -126)


def round_f32(x):
    """Round to the nearest fp32 value (ties to even)."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def rho(x, precision: str):
    """The layer's rounding point for a storage precision."""
    if precision == "f64":
        return np.asarray(x, dtype=np.float64)
    if precision == "f32":
        return round_f32(x)
    if precision in ("bf16", "nvfp4"):
        return round_bf16(x)
    raise ValueError(precision)


# ----------------------------------------------------------------------------
# NVFP4 number formats (E2M1 elements, E4M3 block scales)
# ----------------------------------------------------------------------------

# E2M1: 1 sign, 2 exponent (bias 1), 1 mantissa bit. Magnitude by code 0..7.
E2M1_MAG = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e2m1_decode(code) -> np.ndarray:
    code = np.asarray(code, dtype=np.int64)
    mag = E2M1_MAG[code & 7]
    return np.where(code & 8, -mag, mag)


def e4m3_decode(code) -> np.ndarray:
    """OCP E4M3 ("fn"): bias 7, no infinities, 0x7F/0xFF are NaN."""
    code = np.asarray(code, dtype=np.int64)
    s = (code >> 7) & 1
    e = (code >> 3) & 15
    f = code & 7
    mag = np.where(e == 0, f * 2.0 ** -9, (1.0 + f / 8.0) * np.ldexp(1.0, e - 7))
    mag = np.where((e == 15) & (f == 7), np.nan, mag)
    return np.where(s == 1, -mag, mag)


E4M3_MAG = e4m3_decode(np.arange(127))          # codes 0..126, all finite, ascending


def _nearest_code_rne(v_abs: np.ndarray, table: np.ndarray) -> np.ndarray:
    """Index of the nearest entry of an ascending table; ties go to the even
    index (round to nearest even); beyond the last entry saturates to it."""
    v_abs = np.asarray(v_abs, dtype=np.float64)
    hi = np.searchsorted(table, v_abs, side="left")           # table[hi-1] < v <= table[hi]
    hi = np.clip(hi, 1, len(table) - 1)
    lo = hi - 1
    d_lo = v_abs - table[lo]
    d_hi = table[hi] - v_abs
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    idx = np.where(pick_hi, hi, lo)
    idx = np.where(v_abs >= table[-1], len(table) - 1, idx)  # satfinite
    idx = np.where(v_abs <= table[0], 0, idx)
    return idx.astype(np.int64)


def e2m1_encode(v) -> np.ndarray:
    """Float -> E2M1 code (round to nearest even, saturating). The sign bit is
    the sign of v, also when the magnitude rounds to zero."""
    v = np.asarray(v, dtype=np.float64)
    code = _nearest_code_rne(np.abs(v), E2M1_MAG)
    return (code | np.where(np.signbit(v), 8, 0)).astype(np.uint8)


def e4m3_encode(v) -> np.ndarray:
    """Float -> E4M3 code (round to nearest even, saturating to 448)."""
    v = np.asarray(v, dtype=np.float64)
    code = _nearest_code_rne(np.abs(v), E4M3_MAG)
    return (code | np.where(np.signbit(v), 128, 0)).astype(np.uint8)


NVFP4_BLOCK = 16
E2M1_MAX = 6.0
E4M3_MAX = 448.0


def nvfp4_global_scale(X) -> float:
    """Per-tensor FP32 global scale: fp32(amax / (6 * 448)); 1 when amax is 0."""
    amax = float(np.max(np.abs(X))) if np.size(X) else 0.0
    if amax == 0.0:
        return 1.0
    return float(round_f32(amax / round_f32(E2M1_MAX * E4M3_MAX)))


def nvfp4_quantize(X, s_g: float | None = None):
    """Two-level NVFP4 quantisation of a row-major matrix along its rows.

    X: [rows, cols] float64 values (cols a multiple of 16), each exactly an fp32.
    Returns (codes [rows, cols/2] uint8 -- element 2j in the low nibble, 2j+1 in
    the high nibble; scales [rows, cols/16] uint8 E4M3 codes; s_g float).
    """
    X = np.asarray(X, dtype=np.float64)
    rows, cols = X.shape
    assert cols % NVFP4_BLOCK == 0
    if s_g is None:
        s_g = nvfp4_global_scale(X)
    s_g = float(round_f32(s_g))
    blocks = X.reshape(rows, cols // NVFP4_BLOCK, NVFP4_BLOCK)
    amax_b = np.max(np.abs(blocks), axis=2)
    t = round_f32(s_g * E2M1_MAX)
    r = round_f32(amax_b / t)
    sb_code = e4m3_encode(r)
    sb = e4m3_decode(sb_code)
    sc = round_f32(sb * s_g)
    with np.errstate(divide="ignore", invalid="ignore"):
        v = round_f32(blocks / sc[..., None])
    q = e2m1_encode(v)
    q = np.where((sb == 0.0)[..., None], np.uint8(0), q).astype(np.uint8)
    q = q.reshape(rows, cols)
    codes = (q[:, 0::2] | (q[:, 1::2] << 4)).astype(np.uint8)
    return codes, sb_code, s_g


def nvfp4_quantize_2d(X, s_g: float | None = None):
    """NVFP4 with two-dimensional weight blocks: one E4M3 scale per 16 rows x
    16 columns (greeksharifa page, section 2.4 "NVFP4 Training": the recipe
    scales weights in two-dimensional blocks; the block size is read as the
    16-element micro-block squared, so that W and W^T quantise alike).

    The block amax runs over the block's 256 elements (rows past the end of
    X count as 0); every other step is nvfp4_quantize's. The scale is written
    to each of the block's rows, so the result has nvfp4_quantize's layout
    (codes [rows, cols/2], scales [rows, cols/16]) and decodes the same way.
    """
    X = np.asarray(X, dtype=np.float64)
    rows, cols = X.shape
    assert cols % NVFP4_BLOCK == 0
    if s_g is None:
        s_g = nvfp4_global_scale(X)
    s_g = float(round_f32(s_g))
    nrb = -(-rows // NVFP4_BLOCK)
    Xp = np.zeros((nrb * NVFP4_BLOCK, cols))
    Xp[:rows] = X
    amax_2d = np.max(np.abs(Xp.reshape(nrb, NVFP4_BLOCK, cols // NVFP4_BLOCK, NVFP4_BLOCK)), axis=(1, 3))
    t = round_f32(s_g * E2M1_MAX)
    sb_code_2d = e4m3_encode(round_f32(amax_2d / t))
    sb_code = np.repeat(sb_code_2d, NVFP4_BLOCK, axis=0)[:rows]      # [rows, cols/16]
    sb = e4m3_decode(sb_code)
    sc = round_f32(sb * s_g)
    blocks = X.reshape(rows, cols // NVFP4_BLOCK, NVFP4_BLOCK)
    with np.errstate(divide="ignore", invalid="ignore"):
        v = round_f32(blocks / sc[..., None])
    q = e2m1_encode(v)
    q = np.where((sb == 0.0)[..., None], np.uint8(0), q).astype(np.uint8).reshape(rows, cols)
    codes = (q[:, 0::2] | (q[:, 1::2] << 4)).astype(np.uint8)
    return codes, sb_code.astype(np.uint8), s_g


def nvfp4_unpack(codes) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.uint8)
    out = np.empty(codes.shape[:-1] + (codes.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = codes & 15
    out[..., 1::2] = codes >> 4
    return out


def nvfp4_dequantize(codes, scales, s_g: float) -> np.ndarray:
    """x_hat = e2m1(q) * e4m3(s_b) * s_g, exact in fp64."""
    q = e2m1_decode(nvfp4_unpack(codes))
    rows, cols = q.shape
    sb = e4m3_decode(scales)
    return (q.reshape(rows, cols // NVFP4_BLOCK, NVFP4_BLOCK) * sb[..., None] * s_g).reshape(rows, cols)


def nvfp4_fake_quant(X, s_g: float | None = None):
    codes, sf, s_g = nvfp4_quantize(X, s_g)
    return nvfp4_dequantize(codes, sf, s_g), s_g


# ----------------------------------------------------------------------------
# Routing
# ----------------------------------------------------------------------------


# ----------------------------------------------------------------------------
# FP8 (E4M3) with per-tensor FP32 scales: the shared experts of the Ultra
# checkpoint recipe (chathome page on Nemotron 3 Ultra, quantisation
# paragraph: NVFP4 routed experts next to FP8 shared experts; jiwasawa blog on
# Nemotron 3 Nano, FP8 section: post-training quantisation of weights and
# activations to FP8). The pages give the format only; the reading taken:
# one FP32 scale per weight tensor, amax / 448, and static per-layer FP32
# scales for the two activations (the shared experts' input x and their
# hidden layer), as an inference checkpoint carries them.
# ----------------------------------------------------------------------------

def fp8_scale(X) -> float:
    """Per-tensor FP32 scale of a weight tensor: fp32(amax / 448); 1 when amax is 0."""
    amax = float(np.max(np.abs(X))) if np.size(X) else 0.0
    if amax == 0.0:
        return 1.0
    return float(round_f32(amax / E4M3_MAX))


def fp8_quantize(X, s: float) -> np.ndarray:
    """E4M3 codes of X / s: E4M3_rn_satfinite(fp32(x / s)), s an fp32 value.
    The division is an fp32 operation, emulated exactly (fp64 then fp32)."""
    return e4m3_encode(round_f32(np.asarray(X, dtype=np.float64) / s))


def fp8_dequantize(codes, s: float) -> np.ndarray:
    """x_hat = e4m3(q) * s, exact in fp64."""
    return e4m3_decode(codes) * s


def fp8_fake_quant(X, s: float) -> np.ndarray:
    return fp8_dequantize(fp8_quantize(X, s), s)


def shared_experts_fp8(x, ws1, ws2, s_x: float, s_h: float):
    """Sum over the S shared experts of hs_s Ws2_s^T with FP8 operands.

    x [T, d]; ws1 [S, m_s, d] and ws2 [S, d, m_s] (fp64 values of the stored
    BF16 weights). Each weight tensor (all S experts' Ws1 as one tensor, all
    their Ws2 as another) is quantised with its own amax scale; x with the
    static scale s_x; the hidden layer hs = relu(x_hat Ws1_hat^T)^2 is stored
    as FP8 with the static scale s_h (its rounding point). Returns (sum
    [T, d], hs codes [T, S*m_s], (s_w1, s_w2))."""
    S, ms, d = ws1.shape
    w1 = ws1.reshape(S * ms, d)
    s_w1, s_w2 = fp8_scale(w1), fp8_scale(ws2)
    xq = fp8_fake_quant(x, s_x)
    w1q = fp8_fake_quant(w1, s_w1)
    w2q = fp8_fake_quant(ws2, s_w2)
    h_codes = fp8_quantize(sq_relu(xq @ w1q.T), s_h)
    hs = fp8_dequantize(h_codes, s_h)
    out = np.zeros((x.shape[0], d))
    for s in range(S):
        out += hs[:, s * ms:(s + 1) * ms] @ w2q[s].T
    return out, h_codes, (s_w1, s_w2)


def router_logits(x, w_router, bias=None) -> np.ndarray:
    """logits[t, e] = x_t . W_r[e] (+ b[e]); the gate reads the d-dim x."""
    logits = np.asarray(x, dtype=np.float64) @ np.asarray(w_router, dtype=np.float64).T
    if bias is not None:
        logits = logits + np.asarray(bias, dtype=np.float64)[None, :]
    return logits


def route_topk(logits, K: int):
    """Top-K experts per token, ordered by (logit desc, index asc), and their
    gates: softmax over all N experts restricted to the chosen K, renormalised.

    Returns idx [T, K] int32 (selection order) and gates [T, K] float64.
    """
    logits = np.asarray(logits, dtype=np.float64)
    order = np.argsort(-logits, axis=1, kind="stable")   # stable: lower index first on ties
    idx = order[:, :K].astype(np.int32)
    lmax = np.max(logits, axis=1, keepdims=True)
    p = np.exp(logits - lmax)
    p = p / np.sum(p, axis=1, keepdims=True)             # softmax over all N
    sel = np.take_along_axis(p, idx.astype(np.int64), axis=1)
    gates = sel / np.sum(sel, axis=1, keepdims=True)      # renormalise over the K
    return idx, gates


def near_tie_tokens(logits, K: int, gap: float = 1e-5) -> np.ndarray:
    """Tokens whose routing output is decided by a logit gap below ``gap``:
    two consecutive values among the K+1 largest logits (the K-th against the
    (K+1)-th decides the chosen set; consecutive chosen ones decide their
    order in the output) differ by less than ``gap``."""
    logits = np.asarray(logits, dtype=np.float64)
    s = -np.sort(-logits, axis=1)
    top = s[:, :min(K + 1, logits.shape[1])]
    if top.shape[1] < 2:
        return np.zeros(logits.shape[0], dtype=bool)
    return np.min(top[:, :-1] - top[:, 1:], axis=1) < gap


# ----------------------------------------------------------------------------
# Permutation (dispatch grouped by expert)
# ----------------------------------------------------------------------------


def permute(idx, N: int):
    """Group the flat slots f = t*K + k by expert, stably (expert asc, then f asc).

    Returns counts [N], offsets [N+1], perm_src [T*K] (permuted row r holds slot
    perm_src[r]) and inv_perm [T*K] (slot f sits at permuted row inv_perm[f]).
    """
    flat = np.asarray(idx, dtype=np.int64).reshape(-1)
    counts = np.bincount(flat, minlength=N).astype(np.int32)
    offsets = np.zeros(N + 1, dtype=np.int32)
    np.cumsum(counts, out=offsets[1:])
    perm_src = np.argsort(flat, kind="stable").astype(np.int32)
    inv_perm = np.empty_like(perm_src)
    inv_perm[perm_src] = np.arange(flat.size, dtype=np.int32)
    return counts, offsets, perm_src, inv_perm


# ----------------------------------------------------------------------------
# The layer
# ----------------------------------------------------------------------------


def sq_relu(h):
    return np.square(np.maximum(h, 0.0))


def weights_view(wl, inp, cache: bool = False) -> _Weights:
    """The weights object ``forward`` uses; pass one with cache=True to several
    calls on the same inputs to quantise each NVFP4 expert matrix once."""
    return _Weights(wl, inp, cache)


def quantize_expert_weights(w_bf16_f64: np.ndarray):
    """NVFP4 codes, scales and per-matrix global scale of each expert matrix
    [N, rows, cols] (blocks along the contraction dim, i.e. along cols)."""
    out = []
    for e in range(w_bf16_f64.shape[0]):
        out.append(nvfp4_quantize(w_bf16_f64[e]))
    return out


class _Weights:
    """fp64 views of the stored weights, converted expert by expert on demand.
    With cache=True the NVFP4 quantisation of each expert matrix (codes,
    scales, global scale) is kept, so repeated calls only dequantise."""

    def __init__(self, wl, inp, cache: bool = False):
        self.wl = wl
        self.inp = inp
        self.st = "f32" if wl.dtype == "f32" else "bf16"
        self._q = {} if cache else None

    def dense(self, key):
        return to_f64(self.inp[key], self.st)

    def expert(self, key, e):
        """fp64 values of expert e's matrix as the GEMM sees them."""
        if self.wl.dtype == "nvfp4":
            quant = nvfp4_quantize_2d if getattr(self.wl, "w_block2d", False) else nvfp4_quantize
            if self._q is not None:
                if (key, e) not in self._q:
                    self._q[(key, e)] = quant(to_f64(self.inp[key][e], self.st))
                return nvfp4_dequantize(*self._q[(key, e)])
            return nvfp4_dequantize(*quant(to_f64(self.inp[key][e], self.st)))
        return to_f64(self.inp[key][e], self.st)


def forward(wl, inp, tokens=None, idx_override=None, precision: str | None = None,
            weights: _Weights | None = None, z_rows=None) -> dict:
    """One LatentMoE layer forward.

    wl: a ``lmoe_inputs.Workload``; inp: ``lmoe_inputs.make_inputs(wl)``.
    tokens: optional subset of token indices (tokens are independent, so the
      outputs of a subset equal those rows of the full forward). The NVFP4
      global scale of z is still taken over all T tokens.
    idx_override: optional [len(tokens), K] expert choice (e.g. the GPU's
      choice on documented near-ties); the gates follow the override.
    z_rows: NVFP4 only, optional [len(tokens), l] BF16-valued latent rows to
      quantise instead of the rounded down-projection (an alternative rounding
      of a documented rounding near-tie); the global scale stays the one of
      the full z.
    precision: "f64" (no rounding points), else the workload's own
      ("f32" | "bf16" | "nvfp4").

    Returns a dict with logits, idx, gates, z, counts, offsets, perm_src,
    inv_perm, a (permuted rows), y (permuted rows), c, out, all fp64 except
    the integer buffers.
    """
    prec = precision or wl.dtype
    W = weights or _Weights(wl, inp)
    st = W.st
    x_all = to_f64(inp["x"], st)
    tok = np.arange(wl.T) if tokens is None else np.asarray(tokens)
    x = x_all[tok]
    T = x.shape[0]
    K = wl.K

    # router on the d-dim hidden state
    bias = inp.get("router_bias")
    logits = router_logits(x, W.dense("w_router"), bias)
    idx, gates = route_topk(logits, K)
    if idx_override is not None:
        idx = np.asarray(idx_override, dtype=np.int32)
        lmax = np.max(logits, axis=1, keepdims=True)
        p = np.exp(logits - lmax)
        sel = np.take_along_axis(p, idx.astype(np.int64), axis=1)
        gates = sel / np.sum(sel, axis=1, keepdims=True)

    # down projection d -> l (skipped with identity projections)
    if wl.identity:
        z = x.copy()
        zq_scale = None
    else:
        w_down = W.dense("w_down")
        if prec == "nvfp4":
            z_full = round_bf16(x_all @ w_down.T)
            zq_scale = nvfp4_global_scale(z_full)
            zsel = z_full[tok] if z_rows is None else np.asarray(z_rows, dtype=np.float64)
            z = nvfp4_fake_quant(zsel, zq_scale)[0]
        else:
            z = rho(x @ w_down.T, prec)
            zq_scale = None

    # dispatch grouped by expert
    counts, offsets, perm_src, inv_perm = permute(idx, wl.N)
    rows_tok = perm_src // K
    rows_k = perm_src % K
    l, m = wl.l, wl.m
    a = np.zeros((T * K, m))
    y = np.zeros((T * K, l))
    a_gs = inp.get("a_global_scale")
    for e in range(wl.N):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r0 == r1:
            continue
        ze = z[rows_tok[r0:r1]]
        h = ze @ W.expert("w1", e).T
        if prec == "nvfp4":
            ae = nvfp4_fake_quant(sq_relu(h), a_gs)[0]
        else:
            ae = rho(sq_relu(h), prec)
        a[r0:r1] = ae
        g = gates[rows_tok[r0:r1], rows_k[r0:r1]]
        y[r0:r1] = rho(g[:, None] * (ae @ W.expert("w2", e).T), prec)

    # gate-weighted combine (gates already applied to y)
    c = np.zeros((T, l))
    for k in range(K):
        c += y[inv_perm[np.arange(T) * K + k]]
    c = rho(c, prec)

    # up projection l -> d, plus always-on shared experts on the d-dim x
    if wl.identity:
        out = c.copy()
    else:
        out = c @ W.dense("w_up").T
    if wl.n_shared and getattr(wl, "shared_fp8", False) and prec != "f64":
        ys, _, _ = shared_experts_fp8(x, to_f64(inp["ws1"], st), to_f64(inp["ws2"], st),
                                      inp["shared_x_scale"], inp["shared_h_scale"])
        out = out + ys
    elif wl.n_shared:
        for s in range(wl.n_shared):
            ws1 = to_f64(inp["ws1"][s], st)
            ws2 = to_f64(inp["ws2"][s], st)
            hs = rho(sq_relu(x @ ws1.T), prec)
            out = out + hs @ ws2.T
    out_unrounded = out
    out = rho(out, prec)
    return dict(logits=logits, idx=idx, gates=gates, z=z, z_global_scale=zq_scale,
                counts=counts, offsets=offsets, perm_src=perm_src, inv_perm=inv_perm,
                a=a, y=y, c=c, out=out, out_unrounded=out_unrounded, tokens=tok)


def brute_force_topk(logits_row, K: int):
    """Reference selection by enumerating every K-subset: the subset with the
    largest logit sum, ties broken by the lexicographically smallest sorted
    index tuple; returned in (logit desc, index asc) order. Tiny N only."""
    best = None
    N = len(logits_row)
    for sub in itertools.combinations(range(N), K):
        s = sum(logits_row[i] for i in sub)
        if best is None or s > best[0] or (s == best[0] and sub < best[1]):
            best = (s, sub)
    sel = sorted(best[1], key=lambda i: (-logits_row[i], i))
    return sel
