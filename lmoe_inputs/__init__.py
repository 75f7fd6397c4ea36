"""Seeded synthetic inputs for the LatentMoE layer forward.

This module is shared by the CPU oracle and the CUDA path. It only draws
random numbers and stores them in the number format a workload asks for; it
holds none of the layer's arithmetic (no routing, no projection, no
quantisation).

Workloads (shapes from the Nemotron 3 LatentMoE description: the Ultra-width
LatentMoE uses d=8192, l=2048, 512 experts with 22 active; the standard-MoE
limit uses l=d with 128 experts, 6 active and two always-on shared experts):

* ``tiny_f32``        T=64,    d=256,  l=64,   N=32,  K=4,  m=128, fp32
* ``std_moe_bf16``    T=4096,  d=l=2688 (identity projections), N=128, K=6,
                      m=1856, 2 shared experts of width 1856, BF16
* ``ultra_decode``    T=32,    d=8192, l=2048, N=512, K=22, m=1024, BF16
* ``ultra_zipf``      T=16384, same shapes, additive Zipf(1.1) router bias
* ``ultra_nvfp4``     T=8192,  same shapes, NVFP4 experts and latent
                      activations, 0.1% of x scaled by 50
* ``ultra_decode_nvfp4`` T=32, the same NVFP4 layer in decode

Recipe (every tensor from its own ``SeedSequence`` child, so generation order
and thread count do not change any value):

* x ~ N(0, 1); every weight matrix [out, in] ~ N(0, 1/in).
* Values are drawn in float64 and stored as BF16 bit patterns (``np.uint16``,
  round to nearest even through float32) or as float32 for fp32 workloads.
* Zipf bias: a seeded random permutation pi of the experts and
  b[pi(r)] = -1.1 * ln(r), r = 1..N (a Zipf(1.1) prior in logit space).
* Outliers: exactly round(0.001 * T * d) entries of x, chosen uniformly without
  replacement, multiplied by 50 before storage.
* NVFP4 workloads also carry ``a_global_scale``: the static per-layer FP32
  scale of the FFN hidden activation a = relu(h)^2, as an inference checkpoint
  carries it. Its synthetic value covers |h| <= 16 (a <= 256): 256 / (6 * 448).
* Workloads with FP8 shared experts carry two static per-layer FP32 scales
  the same way: ``shared_x_scale`` = 256 / 448 for the shared experts' input x
  (covers |x| <= 256, the outliers included) and ``shared_h_scale`` = 512 / 448
  for their hidden layer (covers values up to 512).
* ``ultra_nvfp4_fp8shared`` T=8192, the NVFP4 layer with two always-on shared
  experts of width 1024 in FP8 (the Ultra checkpoint recipe: NVFP4 routed,
  FP8 shared experts)
"""
from __future__ import annotations

import concurrent.futures as _cf
import os
from dataclasses import dataclass, replace, asdict

import numpy as np

__all__ = ["Workload", "WORKLOADS", "make_inputs", "bf16_bits", "reduced", "replace"]


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    l: int
    N: int
    K: int
    m: int
    n_shared: int = 0
    m_shared: int = 0
    dtype: str = "bf16"          # "f32" | "bf16" | "nvfp4" (nvfp4: experts + latent acts)
    identity: bool = False       # l == d, no down/up projection
    zipf_bias: bool = False
    outliers: bool = False
    w_block2d: bool = False      # nvfp4: expert weights scaled in 16 x 16 blocks
    shared_fp8: bool = False     # shared experts in FP8 (E4M3, per-tensor scales)
    seed: int = 0

    def as_dict(self):
        return asdict(self)


WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", T=64, d=256, l=64, N=32, K=4, m=128, dtype="f32"),
    "std_moe_bf16": Workload("std_moe_bf16", T=4096, d=2688, l=2688, N=128, K=6, m=1856,
                             n_shared=2, m_shared=1856, dtype="bf16", identity=True),
    "ultra_decode": Workload("ultra_decode", T=32, d=8192, l=2048, N=512, K=22, m=1024,
                             dtype="bf16"),
    "ultra_zipf": Workload("ultra_zipf", T=16384, d=8192, l=2048, N=512, K=22, m=1024,
                           dtype="bf16", zipf_bias=True),
    "ultra_nvfp4": Workload("ultra_nvfp4", T=8192, d=8192, l=2048, N=512, K=22, m=1024,
                            dtype="nvfp4", outliers=True),
    "ultra_decode_nvfp4": Workload("ultra_decode_nvfp4", T=32, d=8192, l=2048, N=512, K=22, m=1024,
                                   dtype="nvfp4", outliers=True),
    "ultra_nvfp4_fp8shared": Workload("ultra_nvfp4_fp8shared", T=8192, d=8192, l=2048, N=512, K=22, m=1024,
                                      n_shared=2, m_shared=1024, dtype="nvfp4", outliers=True,
                                      shared_fp8=True),
}


def reduced(name: str, **sizes) -> Workload:
    """A workload with the structure of ``name`` and smaller sizes."""
    wl = WORKLOADS[name]
    return replace(wl, name=f"{name}_reduced", **sizes)


def bf16_bits(v: np.ndarray) -> np.ndarray:
    """Store float64 values as BF16 bit patterns (nearest even, via float32)."""
    f = np.ascontiguousarray(v, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    u = (u + 0x7FFF + lsb) >> 16
    return u.astype(np.uint16)


# Fixed spawn order of the top-level children; never reorder.
_STREAMS = ("x", "w_router", "w_down", "w1", "w2", "w_up", "ws1", "ws2", "bias_perm", "outliers")


def _normal(ss: np.random.SeedSequence, shape, std: float) -> np.ndarray:
    return np.random.Generator(np.random.PCG64(ss)).standard_normal(shape) * std


def _store(v: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "f32":
        return v.astype(np.float32)
    return bf16_bits(v)


def _stacked(ss: np.random.SeedSequence, count: int, rows: int, cols: int, dtype: str,
             pool) -> np.ndarray:
    """[count, rows, cols] matrices, each ~N(0, 1/cols), one child seed per matrix."""
    out = np.empty((count, rows, cols), dtype=np.float32 if dtype == "f32" else np.uint16)
    kids = ss.spawn(count)
    std = 1.0 / np.sqrt(cols)

    def one(e):
        out[e] = _store(_normal(kids[e], (rows, cols), std), dtype)

    list(pool.map(one, range(count)))
    return out


def make_inputs(wl: Workload, threads: int | None = None) -> dict:
    """All inputs of one layer forward, as numpy arrays.

    BF16 tensors are ``np.uint16`` bit patterns; fp32 tensors are ``np.float32``.
    Keys: x [T,d], w_router [N,d], router_bias [N] f32 or None, w_down [l,d] or
    None, w_up [d,l] or None, w1 [N,m,l], w2 [N,l,m], ws1 [S,m_s,d] or None,
    ws2 [S,d,m_s] or None, a_global_scale (float or None).
    NVFP4 workloads hold their expert weights here in BF16; quantising them is
    part of the method, done by each side itself.
    """
    kids = dict(zip(_STREAMS, np.random.SeedSequence(wl.seed).spawn(len(_STREAMS))))
    st = "f32" if wl.dtype == "f32" else "bf16"
    threads = threads or min(16, len(os.sched_getaffinity(0)))
    with _cf.ThreadPoolExecutor(threads) as pool:
        x = _normal(kids["x"], (wl.T, wl.d), 1.0)
        if wl.outliers:
            g = np.random.Generator(np.random.PCG64(kids["outliers"]))
            n_out = int(round(0.001 * wl.T * wl.d))
            pos = g.choice(wl.T * wl.d, size=n_out, replace=False)
            x.reshape(-1)[pos] *= 50.0
        inp = {"x": _store(x, st)}
        del x
        inp["w_router"] = _store(_normal(kids["w_router"], (wl.N, wl.d), 1.0 / np.sqrt(wl.d)), st)
        if wl.identity:
            assert wl.l == wl.d
            inp["w_down"] = None
            inp["w_up"] = None
        else:
            inp["w_down"] = _store(_normal(kids["w_down"], (wl.l, wl.d), 1.0 / np.sqrt(wl.d)), st)
            inp["w_up"] = _store(_normal(kids["w_up"], (wl.d, wl.l), 1.0 / np.sqrt(wl.l)), st)
        inp["w1"] = _stacked(kids["w1"], wl.N, wl.m, wl.l, st, pool)
        inp["w2"] = _stacked(kids["w2"], wl.N, wl.l, wl.m, st, pool)
        if wl.n_shared:
            inp["ws1"] = _stacked(kids["ws1"], wl.n_shared, wl.m_shared, wl.d, st, pool)
            inp["ws2"] = _stacked(kids["ws2"], wl.n_shared, wl.d, wl.m_shared, st, pool)
        else:
            inp["ws1"] = None
            inp["ws2"] = None
    if wl.zipf_bias:
        g = np.random.Generator(np.random.PCG64(kids["bias_perm"]))
        perm = g.permutation(wl.N)
        bias = np.empty(wl.N, dtype=np.float64)
        bias[perm] = -1.1 * np.log(np.arange(1, wl.N + 1, dtype=np.float64))
        inp["router_bias"] = bias.astype(np.float32)
    else:
        inp["router_bias"] = None
    inp["a_global_scale"] = (256.0 / (6.0 * 448.0)) if wl.dtype == "nvfp4" else None
    if inp["a_global_scale"] is not None:
        inp["a_global_scale"] = float(np.float32(inp["a_global_scale"]))
    if wl.shared_fp8:
        inp["shared_x_scale"] = float(np.float32(256.0 / 448.0))
        inp["shared_h_scale"] = float(np.float32(512.0 / 448.0))
    else:
        inp["shared_x_scale"] = None
        inp["shared_h_scale"] = None
    return inp
