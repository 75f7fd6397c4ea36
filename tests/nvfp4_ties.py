"""Rounding near-ties of the latent z that decide NVFP4 codes.

z is rounded to BF16 before it is quantised. Where the exact down-projection
lies within a hair of a BF16 rounding midpoint, the GPU (fp32 accumulation)
and the oracle (fp64) may round it to different neighbours; both are correct
roundings, and if the two differ in the NVFP4 code or block scale of their
block, the layer legitimately takes a different quantised input from there on.
For such tokens the GPU output is compared with the oracle run on every
combination of the alternative roundings (the documented near-tie rule for
quantisation decisions)."""
from __future__ import annotations

import itertools

import numpy as np

from oracle import lmoe_oracle as O

EPS = 2.0 ** -16          # relative distance to a rounding midpoint counted as a tie
# The GPU accumulates the down-projection in fp32 on the tensor cores, so its
# result can differ from the exact one by an amount set by the terms of the
# dot product, not by the result: where the terms cancel, a relative window is
# too narrow. The router GEMM's measured logit error on the same hardware is
# about 2^-14 of the L2 norm of its terms (||t||_2 = sqrt(sum_i (x_i w_i)^2)),
# so the window also covers 2^-13 * ||t||_2, twice that.
EPS_L2 = 2.0 ** -13


def z_exact(inp, tokens):
    """Exact down-projection rows and the L2 norms of their dot products' terms."""
    x = O.from_bf16_bits(inp["x"][tokens])
    w = O.from_bf16_bits(inp["w_down"])
    return x @ w.T, np.sqrt((x * x) @ (w * w).T)


def code_changing_ties(zx_row: np.ndarray, s_g: float, tnorm_row=None, eps: float = EPS,
                       eps_l2: float = EPS_L2, kmax: int = 8):
    """[(j, alternative value)] for elements whose other BF16 rounding changes
    the NVFP4 codes or scale of their 16-element block, nearest (relative to
    the window) first, at most kmax."""
    zr = O.round_bf16(zx_row)
    other = O.round_bf16(2.0 * zx_row - zr)          # the neighbour on the other side of the midpoint
    mid = (zr + other) / 2.0
    win = eps * np.abs(zx_row)
    if tnorm_row is not None:
        win = np.maximum(win, eps_l2 * tnorm_row)
    dist = np.abs(zx_row - mid)
    cand = np.where((other != zr) & (dist <= win))[0]
    near = cand[np.argsort(dist[cand] / win[cand], kind="stable")]
    out = []
    c0, s0, _ = O.nvfp4_quantize(zr[None, :], s_g)
    for j in near:
        alt = zr.copy()
        alt[j] = other[j]
        b = j // 16
        c1, s1, _ = O.nvfp4_quantize(alt[None, :], s_g)
        if s1[0, b] != s0[0, b] or np.any(c1[0, b * 8:(b + 1) * 8] != c0[0, b * 8:(b + 1) * 8]):
            out.append((int(j), float(other[j])))
            if len(out) == kmax:
                break
    return zr, out


def variant_rows(zr: np.ndarray, ties, kmax: int = 8):
    """Every combination of alternative roundings (at most 2^kmax rows)."""
    ties = ties[:kmax]
    for mask in itertools.product((0, 1), repeat=len(ties)):
        row = zr.copy()
        for on, (j, v) in zip(mask, ties):
            if on:
                row[j] = v
        yield row
