"""Helpers shared by the GPU parity tests: move seeded inputs to the device,
build the C-ABI config/weights, compare against the oracle."""
from __future__ import annotations

import numpy as np
import torch

import latentmoe_fwd_b200 as L


def to_dev(a, dtype_tag):
    """numpy (BF16 bits as uint16, or float32) -> cuda tensor."""
    if a is None:
        return None
    if dtype_tag == "f32":
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def cfg_of(wl, T=None):
    act = L.F32 if wl.dtype == "f32" else L.BF16
    expert = {"f32": L.F32, "bf16": L.BF16, "nvfp4": L.NVFP4}[wl.dtype]
    return L.config(T=wl.T if T is None else T, d=wl.d, l=wl.l, N=wl.N, K=wl.K, m=wl.m,
                    n_shared=wl.n_shared, m_shared=wl.m_shared, act=act, expert=expert,
                    identity=wl.identity, shared_fp8=getattr(wl, "shared_fp8", False))


def fp8_quantize_dev(x: torch.Tensor, rows: int, cols: int, scale_in=None):
    """lmoe_fp8_quantize on a device tensor: (codes [rows][cols] uint8, scale [1])."""
    codes = torch.empty((rows, cols), dtype=torch.uint8, device="cuda")
    scale = torch.empty(1, dtype=torch.float32, device="cuda")
    ws = L.workspace(L.config(T=rows, d=cols, l=cols, N=1, K=1, m=cols), L.OP_FP8_QUANTIZE)
    dt = L.BF16 if x.dtype == torch.bfloat16 else L.F32
    L.fp8_quantize(x, dt, rows, cols, scale_in, codes, scale, ws)
    torch.cuda.synchronize()
    return codes, scale


def quantize_dev(x: torch.Tensor, rows: int, cols: int, layout=L.SF_ROWMAJOR, global_in=None):
    """lmoe_nvfp4_quantize on a device tensor: (codes, sf, global scale)."""
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device="cuda")
    if (layout & ~L.SF_BLOCK_16X16) == L.SF_MMA_TILED:
        sf = torch.empty((((rows + 127) // 128) * 128 * ((cols + 63) // 64) * 4,), dtype=torch.uint8, device="cuda")
    else:
        sf = torch.empty((rows, cols // 16), dtype=torch.uint8, device="cuda")
    g = torch.empty(1, dtype=torch.float32, device="cuda")
    ws = L.workspace(L.config(T=rows, d=cols, l=cols, N=1, K=1, m=cols), L.OP_NVFP4_QUANTIZE)
    dt = L.BF16 if x.dtype == torch.bfloat16 else L.F32
    L.nvfp4_quantize(x, dt, rows, cols, global_in, codes, sf, g, layout, ws)
    st, info = L.read_device_error(ws)
    assert st == L.OK, (st, info)
    return codes, sf, g


def quantize_experts_dev(w: torch.Tensor, block2d: bool = False):
    """Per-expert NVFP4 weights [N][rows][cols] with MMA-tiled scales (16 x 16
    scale blocks with block2d)."""
    N, rows, cols = w.shape
    codes = torch.empty((N, rows, cols // 2), dtype=torch.uint8, device="cuda")
    sf = torch.empty((N, rows * cols // 16), dtype=torch.uint8, device="cuda")
    gs = torch.empty(N, dtype=torch.float32, device="cuda")
    layout = L.SF_MMA_TILED | (L.SF_BLOCK_16X16 if block2d else 0)
    for e in range(N):
        c, f, g = quantize_dev(w[e], rows, cols, layout)
        codes[e].copy_(c)
        sf[e].copy_(f)
        gs[e:e + 1].copy_(g)
    return codes, sf, gs


class DevLayer:
    """Device copies of one workload's inputs and the C-ABI weight struct."""

    def __init__(self, wl, inp):
        self.wl = wl
        st = "f32" if wl.dtype == "f32" else "bf16"
        self.st = st
        self.x = to_dev(inp["x"], st)
        self.t = {k: to_dev(inp[k], st) for k in ("w_router", "w_down", "w_up", "w1", "w2", "ws1", "ws2")}
        self.bias = None if inp["router_bias"] is None else torch.from_numpy(inp["router_bias"]).cuda()
        self.cfg = cfg_of(wl)
        extra = {}
        if wl.dtype == "nvfp4":
            c1, f1, g1 = quantize_experts_dev(self.t["w1"], wl.w_block2d)
            c2, f2, g2 = quantize_experts_dev(self.t["w2"], wl.w_block2d)
            a_gs = torch.tensor([inp["a_global_scale"]], dtype=torch.float32, device="cuda")
            self.t.update(w1=c1, w2=c2)
            extra = dict(w1_sf=f1, w2_sf=f2, w1_gs=g1, w2_gs=g2, a_global_scale=a_gs)
        if getattr(wl, "shared_fp8", False):
            # each shared weight tensor (all S experts stacked) quantised with its own amax scale
            S, ms, d = wl.n_shared, wl.m_shared, wl.d
            q1, s1 = fp8_quantize_dev(self.t["ws1"].reshape(S * ms, d), S * ms, d)
            q2, s2 = fp8_quantize_dev(self.t["ws2"].reshape(S * d, ms), S * d, ms)
            self.t.update(ws1=q1.reshape(S, ms, d), ws2=q2.reshape(S, d, ms))
            extra.update(ws1_scale=s1, ws2_scale=s2,
                         shared_x_scale=torch.tensor([inp["shared_x_scale"]], dtype=torch.float32, device="cuda"),
                         shared_h_scale=torch.tensor([inp["shared_h_scale"]], dtype=torch.float32, device="cuda"))
        self.w = L.weights(w_router=self.t["w_router"], router_bias=self.bias, w_down=self.t["w_down"],
                           w_up=self.t["w_up"], w1=self.t["w1"], w2=self.t["w2"], ws1=self.t["ws1"],
                           ws2=self.t["ws2"], **extra)

    def forward(self):
        out = torch.empty((self.wl.T, self.wl.d), dtype=self.x.dtype, device="cuda")
        ws = L.workspace(self.cfg, L.OP_FORWARD)
        L.forward(self.cfg, self.w, self.x, out, ws)
        st, info = L.read_device_error(ws)
        assert st == L.OK, (L.status_string(st), hex(info))
        return out

    def route(self):
        T, N, K = self.wl.T, self.wl.N, self.wl.K
        idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
        w = torch.empty((T, K), dtype=torch.float32, device="cuda")
        logits = torch.empty((T, N), dtype=torch.float32, device="cuda")
        ws = L.workspace(self.cfg, L.OP_ROUTE)
        L.route(self.cfg, self.x, self.t["w_router"], self.bias, None, idx, w, logits, ws)
        torch.cuda.synchronize()
        return idx.cpu().numpy(), w.cpu().numpy(), logits.cpu().numpy()


def as_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_max_err(got: np.ndarray, ref: np.ndarray) -> float:
    rms = float(np.sqrt(np.mean(ref ** 2)))
    return float(np.max(np.abs(got - ref))) / rms


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    _, e = np.frexp(np.abs(v))
    e = np.maximum(e - 1, -126)
    return np.ldexp(1.0, e - 7)


def bf16_parity(got: np.ndarray, ref_unrounded: np.ndarray, ref_rounded: np.ndarray):
    """(excess, raw) errors of a BF16 output, both relative to RMS(ref).

    excess: max over elements of |got - exact| beyond half a BF16 step of the
      oracle's value -- the error a BF16 output adds on top of its own
      unavoidable representation error. This is what the 2e-2 * RMS and
      8e-2 * RMS bars are applied to.
    raw: max |got - RN_bf16(oracle)|, reported alongside.
    """
    rms = float(np.sqrt(np.mean(ref_rounded ** 2)))
    excess = np.maximum(0.0, np.abs(got - ref_unrounded) - bf16_ulp(ref_rounded) / 2).max() / rms
    raw = np.abs(got - ref_rounded).max() / rms
    return float(excess), float(raw)


def bf16_raw_within(got: np.ndarray, ref_rounded: np.ndarray, tol: float):
    """Raw bound, element by element: |got - RN_bf16(oracle)| <= tol * RMS + one
    BF16 step of the element. A correct BF16 output can sit one step away
    from the oracle's rounding (its own accumulation rounds on the other side
    of a midpoint), so the step is allowed on top of the output tolerance.
    Returns (all within, max over elements of |err| / bound)."""
    rms = float(np.sqrt(np.mean(ref_rounded ** 2)))
    bound = tol * rms + bf16_ulp(ref_rounded)
    r = np.abs(got - ref_rounded) / bound
    return bool(np.all(r <= 1.0)), float(r.max())
