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


def z_exact(inp, tokens):
    x = O.from_bf16_bits(inp["x"][tokens])
    return x @ O.from_bf16_bits(inp["w_down"]).T


def code_changing_ties(zx_row: np.ndarray, s_g: float, eps: float = EPS):
    """[(j, alternative value)] for elements whose other BF16 rounding changes
    the NVFP4 codes or scale of their 16-element block."""
    zr = O.round_bf16(zx_row)
    other = O.round_bf16(2.0 * zx_row - zr)          # the neighbour on the other side of the midpoint
    mid = (zr + other) / 2.0
    near = np.where((other != zr) & (np.abs(zx_row - mid) <= eps * np.abs(zx_row)))[0]
    out = []
    c0, s0, _ = O.nvfp4_quantize(zr[None, :], s_g)
    for j in near:
        alt = zr.copy()
        alt[j] = other[j]
        b = j // 16
        c1, s1, _ = O.nvfp4_quantize(alt[None, :], s_g)
        if s1[0, b] != s0[0, b] or np.any(c1[0, b * 8:(b + 1) * 8] != c0[0, b * 8:(b + 1) * 8]):
            out.append((int(j), float(other[j])))
    return zr, out


def variant_rows(zr: np.ndarray, ties, kmax: int = 6):
    """Every combination of alternative roundings (at most 2^kmax rows)."""
    ties = ties[:kmax]
    for mask in itertools.product((0, 1), repeat=len(ties)):
        row = zr.copy()
        for on, (j, v) in zip(mask, ties):
            if on:
                row[j] = v
        yield row
