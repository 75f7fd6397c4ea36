"""Python binding of liblmoe.so, the B200 LatentMoE layer-forward library.

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels. PyTorch provides device memory and streams. Importing this package
loads the shared library and fails loudly if it has not been built
(``python latentmoe_fwd_b200/build.py``).

Entry points mirror include/lmoe.h: ``route``, ``permute`` (and
``permute_noalloc``), ``expert_ffn``, ``combine``, ``forward`` (and
``forward_traced``), ``nvfp4_quantize``, ``nvfp4_quantize_ex``, ``nvfp4_transpose_2d``, ``fp8_quantize``,
plus ``workspace_size``,
``padded_rows``, ``workspace``, ``read_device_error``,
``selftest_wait_timeout`` and ``kernel_launch_count``.
Tensor arguments are torch tensors (or None); their ``data_ptr()`` is passed.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
# LMOE_LIBRARY selects another build of the same library (for instance the
# bounds-checking debug build, liblmoe_checks.so); the default is the release build.
LIB_PATH = os.environ.get("LMOE_LIBRARY") or os.path.join(HERE, "liblmoe.so")

# status codes
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_DEVICE_TIMEOUT, ERR_DEVICE_BOUNDS = range(7)
F32, BF16, NVFP4 = 0, 1, 2
SF_ROWMAJOR, SF_MMA_TILED = 0, 1
SF_BLOCK_16X16 = 0x10          # OR into the layout: 16 x 16 scale blocks
QX_TRANSPOSE, QX_RHT, QX_SR = 1, 2, 4   # nvfp4_quantize_ex flags
FLAG_IDENTITY_PROJ = 1
FLAG_SHARED_FP8 = 2            # shared experts in FP8 (E4M3, per-tensor scales)
OP_ROUTE, OP_PERMUTE, OP_EXPERT_FFN, OP_COMBINE, OP_FORWARD, OP_NVFP4_QUANTIZE, OP_FP8_QUANTIZE = range(7)

EXPORTS = ("lmoe_workspace_size", "lmoe_padded_rows", "lmoe_route", "lmoe_permute",
           "lmoe_expert_ffn", "lmoe_combine", "lmoe_forward", "lmoe_nvfp4_quantize",
           "lmoe_read_device_error", "lmoe_status_string", "lmoe_kernel_launch_count",
           "lmoe_forward_traced", "lmoe_permute_noalloc", "lmoe_selftest_wait_timeout", "lmoe_fp8_quantize",
           "lmoe_nvfp4_quantize_ex", "lmoe_nvfp4_quantize_ex_workspace", "lmoe_nvfp4_transpose_2d",
           "lmoe_nvfp4_gemm",
           "lmoe_ep_plan", "lmoe_ep_reorder", "lmoe_ep_slot_bases", "lmoe_ep_dispatch", "lmoe_ep_combine",
           "lmoe_expert_backward_nvfp4",
           "lmoe_expert_backward_nvfp4_workspace", "lmoe_backward_nvfp4", "lmoe_backward_nvfp4_workspace")
TRACE_EVENTS = 8
TRACE_STAGES = ("route", "down_proj", "permute", "expert_gemm1", "expert_gemm2", "combine", "up_proj")


class Config(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("d", ctypes.c_int32), ("l", ctypes.c_int32),
                ("N", ctypes.c_int32), ("K", ctypes.c_int32), ("m", ctypes.c_int32),
                ("n_shared", ctypes.c_int32), ("m_shared", ctypes.c_int32),
                ("act", ctypes.c_int32), ("expert", ctypes.c_int32), ("flags", ctypes.c_uint32)]


class Weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "w_router", "router_bias", "w_down", "w_up", "w1", "w2", "w1_sf", "w2_sf",
        "w1_gs", "w2_gs", "a_global_scale", "ws1", "ws2", "ws1_scale", "ws2_scale", "shared_x_scale",
        "shared_h_scale")]


class Grads(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "dx", "dw_router", "drouter_bias", "dw_down", "dw_up", "dw1", "dw2", "dws1", "dws2")]


class LmoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python latentmoe_fwd_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.c_void_p
    I64 = ctypes.c_int64
    C = ctypes.POINTER(Config)
    W = ctypes.POINTER(Weights)
    sig = {
        "lmoe_workspace_size": (ctypes.c_size_t, [C, ctypes.c_int]),
        "lmoe_padded_rows": (I64, [C]),
        "lmoe_route": (ctypes.c_int, [C, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]),
        "lmoe_permute": (ctypes.c_int, [C, P, P, P, P, P, P, I64, P, P, P, P, P, P, ctypes.c_size_t, P]),
        "lmoe_permute_noalloc": (ctypes.c_int, [C, P, P, P, P, P, P, I64, P, P, P, P, P, P]),
        "lmoe_expert_ffn": (ctypes.c_int, [C, W, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]),
        "lmoe_combine": (ctypes.c_int, [C, P, P, P, P, P, P, P, P]),
        "lmoe_forward": (ctypes.c_int, [C, W, P, P, P, ctypes.c_size_t, P]),
        "lmoe_forward_traced": (ctypes.c_int, [C, W, P, P, P, ctypes.c_size_t, P, ctypes.POINTER(P)]),
        "lmoe_nvfp4_quantize": (ctypes.c_int, [P, ctypes.c_int, I64, I64, P, P, P, P, ctypes.c_int, P,
                                               ctypes.c_size_t, P]),
        "lmoe_read_device_error": (ctypes.c_int, [P, P, ctypes.POINTER(ctypes.c_uint32)]),
        "lmoe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "lmoe_kernel_launch_count": (ctypes.c_uint64, []),
        "lmoe_selftest_wait_timeout": (ctypes.c_int, [P, ctypes.c_size_t, ctypes.c_uint64, P]),
        "lmoe_fp8_quantize": (ctypes.c_int, [P, ctypes.c_int, I64, I64, P, P, P, P, ctypes.c_size_t, P]),
        "lmoe_nvfp4_quantize_ex_workspace": (ctypes.c_size_t, [I64, I64]),
        "lmoe_nvfp4_transpose_2d": (ctypes.c_int, [P, P, I64, I64, I64, P, P, P]),
        "lmoe_ep_plan": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_int] + [P] * 12),
        "lmoe_ep_reorder": (ctypes.c_int, [P, P, I64, ctypes.c_int, P, P, P, I64, P]),
        "lmoe_ep_slot_bases": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, P]),
        "lmoe_ep_dispatch": (ctypes.c_int, [I64, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, I64, P, P, P, P, P, P,
                                            I64, P, P, P, P]),
        "lmoe_ep_combine": (ctypes.c_int, [I64, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, I64, P, P,
                                           P, P, P, P, P, P]),
        "lmoe_nvfp4_gemm": (ctypes.c_int, [ctypes.c_int, P, P, I64, P, P, P, ctypes.c_int, P, P, P, ctypes.c_int,
                                           I64, P, P, I64, P, ctypes.c_size_t, P]),
        "lmoe_nvfp4_quantize_ex": (ctypes.c_int, [P, ctypes.c_int, I64, I64, ctypes.c_uint32, ctypes.c_uint32,
                                                  ctypes.c_uint64, ctypes.c_uint32, P, P, P, P, ctypes.c_int, P,
                                                  ctypes.c_size_t, P]),
        "lmoe_expert_backward_nvfp4_workspace": (ctypes.c_size_t, [C, P]),
        "lmoe_backward_nvfp4_workspace": (ctypes.c_size_t, [C]),
        "lmoe_backward_nvfp4": (ctypes.c_int, [C, W, P, P, P, ctypes.c_uint64, ctypes.c_uint32,
                                               ctypes.POINTER(Grads), P, ctypes.c_size_t, P]),
        "lmoe_expert_backward_nvfp4": (ctypes.c_int, [C, P, P, P, P, P, P, P, P, P, P, P, ctypes.c_uint64,
                                                      ctypes.c_uint32, P, P, P, P, P, ctypes.c_size_t, P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


lib = _load()


def status_string(s: int) -> str:
    return lib.lmoe_status_string(int(s)).decode()


def _p(t):
    """Device pointer of a tensor (or a raw address given as an int), or None.
    A torch tensor in host memory is rejected here: its address would reach a
    kernel as a device pointer."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if getattr(t, "is_cuda", True) is False:
        raise ValueError(f"expected a CUDA tensor, got one on {t.device}")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(st: int, where: str):
    if st != OK:
        raise LmoeError(st, where)


def config(T, d, l, N, K, m, n_shared=0, m_shared=0, act=BF16, expert=BF16, identity=False,
           shared_fp8=False) -> Config:
    flags = (FLAG_IDENTITY_PROJ if identity else 0) | (FLAG_SHARED_FP8 if shared_fp8 else 0)
    return Config(T=T, d=d, l=l, N=N, K=K, m=m, n_shared=n_shared, m_shared=m_shared, act=act,
                  expert=expert, flags=flags)


def weights(**tensors) -> Weights:
    w = Weights()
    for k, v in tensors.items():
        setattr(w, k, _p(v))
    w._keep = tensors   # keep the tensors alive as long as the struct
    return w


def workspace_size(cfg: Config, op: int) -> int:
    return int(lib.lmoe_workspace_size(ctypes.byref(cfg), op))


def padded_rows(cfg: Config) -> int:
    return int(lib.lmoe_padded_rows(ctypes.byref(cfg)))


def kernel_launch_count() -> int:
    return int(lib.lmoe_kernel_launch_count())


def workspace(cfg: Config, op: int, device="cuda"):
    """A workspace tensor for `op`; its error word starts cleared."""
    import torch
    n = workspace_size(cfg, op)
    ws = torch.empty(max(n, 256), dtype=torch.uint8, device=device)
    ws[:256].zero_()
    return ws


def route(cfg, x, w_router, bias, logits_in, topk_idx, topk_w, logits_out, ws, stream=None):
    _check(lib.lmoe_route(ctypes.byref(cfg), _p(x), _p(w_router), _p(bias), _p(logits_in), _p(topk_idx),
                          _p(topk_w), _p(logits_out), _p(ws), ws.numel(), _stream(stream)), "lmoe_route")


def permute(cfg, topk_idx, offsets, perm_src, inv_perm, padded_offsets, rows=None, row_bytes=0,
            permuted_rows=None, rows_sf=None, permuted_sf=None, topk_w=None, perm_gate=None, ws=None,
            stream=None):
    _check(lib.lmoe_permute(ctypes.byref(cfg), _p(topk_idx), _p(offsets), _p(perm_src), _p(inv_perm),
                            _p(padded_offsets), _p(rows), int(row_bytes), _p(permuted_rows), _p(rows_sf),
                            _p(permuted_sf), _p(topk_w), _p(perm_gate), _p(ws), ws.numel(),
                            _stream(stream)), "lmoe_permute")


def permute_noalloc(cfg, topk_idx, offsets, perm_src, inv_perm, padded_offsets, rows=None, row_bytes=0,
                    permuted_rows=None, rows_sf=None, permuted_sf=None, topk_w=None, perm_gate=None,
                    stream=None):
    """lmoe_permute without a workspace (the library's fixed scratch array is
    used instead), for callers that may not allocate device memory."""
    _check(lib.lmoe_permute_noalloc(ctypes.byref(cfg), _p(topk_idx), _p(offsets), _p(perm_src), _p(inv_perm),
                                    _p(padded_offsets), _p(rows), int(row_bytes), _p(permuted_rows),
                                    _p(rows_sf), _p(permuted_sf), _p(topk_w), _p(perm_gate), _stream(stream)),
           "lmoe_permute_noalloc")


def expert_ffn(cfg, w: Weights, permuted_in, permuted_sf, in_global_scale, offsets, padded_offsets,
               perm_gate, y_perm, ws, stream=None):
    _check(lib.lmoe_expert_ffn(ctypes.byref(cfg), ctypes.byref(w), _p(permuted_in), _p(permuted_sf),
                               _p(in_global_scale), _p(offsets), _p(padded_offsets), _p(perm_gate),
                               _p(y_perm), _p(ws), ws.numel(), _stream(stream)), "lmoe_expert_ffn")


def combine(cfg, y_perm, topk_idx, inv_perm, offsets, padded_offsets, topk_w, c, stream=None):
    _check(lib.lmoe_combine(ctypes.byref(cfg), _p(y_perm), _p(topk_idx), _p(inv_perm), _p(offsets),
                            _p(padded_offsets), _p(topk_w), _p(c), _stream(stream)), "lmoe_combine")


def forward(cfg, w: Weights, x, out, ws, stream=None):
    _check(lib.lmoe_forward(ctypes.byref(cfg), ctypes.byref(w), _p(x), _p(out), _p(ws), ws.numel(),
                            _stream(stream)), "lmoe_forward")


def forward_traced(cfg, w: Weights, x, out, ws, events, stream=None):
    """lmoe_forward recording ``TRACE_EVENTS`` torch.cuda.Event objects (timing
    enabled) at the stage boundaries on the launch stream."""
    assert len(events) == TRACE_EVENTS
    for e in events:
        if e.cuda_event == 0:      # torch creates the CUDA event on its first record
            e.record()
    arr = (ctypes.c_void_p * TRACE_EVENTS)(*[e.cuda_event for e in events])
    _check(lib.lmoe_forward_traced(ctypes.byref(cfg), ctypes.byref(w), _p(x), _p(out), _p(ws), ws.numel(),
                                   _stream(stream), arr), "lmoe_forward_traced")


def nvfp4_quantize(x, in_dtype, rows, cols, global_in, codes, sf, global_out, sf_layout, ws, stream=None):
    _check(lib.lmoe_nvfp4_quantize(_p(x), int(in_dtype), int(rows), int(cols), _p(global_in), _p(codes),
                                   _p(sf), _p(global_out), int(sf_layout), _p(ws), ws.numel(),
                                   _stream(stream)), "lmoe_nvfp4_quantize")


def fp8_quantize(x, in_dtype, rows, cols, scale_in, codes, scale_out, ws=None, stream=None):
    """lmoe_fp8_quantize: E4M3 codes of x / s with one FP32 scale per tensor
    (scale_in, or amax / 448 when scale_in is None; scale_out receives it)."""
    _check(lib.lmoe_fp8_quantize(_p(x), int(in_dtype), int(rows), int(cols), _p(scale_in), _p(codes),
                                 _p(scale_out), _p(ws), 0 if ws is None else ws.numel(), _stream(stream)),
           "lmoe_fp8_quantize")


def nvfp4_quantize_ex(x, in_dtype, rows, cols, flags, rht_signs, seed, sr_stream, global_in, codes, sf, global_out,
                      sf_layout, ws=None, stream=None):
    """lmoe_nvfp4_quantize_ex: the training recipe's NVFP4 quantiser (transpose,
    random Hadamard transform, stochastic rounding; see the header)."""
    if ws is None and global_in is None:
        import torch
        ws = torch.zeros(int(lib.lmoe_nvfp4_quantize_ex_workspace(int(rows), int(cols))), dtype=torch.uint8,
                         device="cuda")
    _check(lib.lmoe_nvfp4_quantize_ex(_p(x), int(in_dtype), int(rows), int(cols), int(flags), int(rht_signs),
                                      int(seed), int(sr_stream), _p(global_in), _p(codes), _p(sf), _p(global_out),
                                      int(sf_layout), _p(ws), 0 if ws is None else ws.numel(), _stream(stream)),
           "lmoe_nvfp4_quantize_ex")


def nvfp4_transpose_2d(codes, sf, groups, rows, cols, codes_t, sf_t, stream=None):
    """lmoe_nvfp4_transpose_2d: codes and MMA-tiled scales of NVFP4 matrices
    with 16 x 16 blocks -> those of their transposes."""
    _check(lib.lmoe_nvfp4_transpose_2d(_p(codes), _p(sf), int(groups), int(rows), int(cols), _p(codes_t), _p(sf_t),
                                       _stream(stream)), "lmoe_nvfp4_transpose_2d")


def nvfp4_gemm(groups, offsets, padded_offsets, a_rows, a_codes, a_sf, a_global, a_global_per_group, b_codes, b_sf,
               b_global, cols, k, row_scale, out, ld_out, ws, stream=None):
    """lmoe_nvfp4_gemm: grouped block-scaled NVFP4 GEMM with a BF16 result."""
    _check(lib.lmoe_nvfp4_gemm(int(groups), _p(offsets), _p(padded_offsets), int(a_rows), _p(a_codes), _p(a_sf),
                               _p(a_global), int(a_global_per_group), _p(b_codes), _p(b_sf), _p(b_global),
                               int(cols), int(k), _p(row_scale), _p(out), int(ld_out), _p(ws), ws.numel(),
                               _stream(stream)), "lmoe_nvfp4_gemm")


def expert_backward_nvfp4_workspace(cfg: Config, counts) -> int:
    """lmoe_expert_backward_nvfp4_workspace (counts: host int32 array [N])."""
    import numpy as np
    counts = np.ascontiguousarray(counts, dtype=np.int32)
    return int(lib.lmoe_expert_backward_nvfp4_workspace(ctypes.byref(cfg),
                                                        counts.ctypes.data_as(ctypes.c_void_p)))


def expert_backward_nvfp4(cfg: Config, counts, offsets, padded_offsets, z_codes, z_sf, z_global, w1, w2, a_global,
                          gate, dy, seed, rht_signs, dz, dgate, dw1, dw2, ws=None, stream=None):
    """lmoe_expert_backward_nvfp4: the routed experts' backward under the NVFP4
    training recipe (see the header). counts: host int32 array [N]; the rest
    device tensors. Allocates the workspace when none is given."""
    import numpy as np
    counts = np.ascontiguousarray(counts, dtype=np.int32)
    if ws is None:
        import torch
        ws = torch.zeros(expert_backward_nvfp4_workspace(cfg, counts), dtype=torch.uint8, device="cuda")
    _check(lib.lmoe_expert_backward_nvfp4(ctypes.byref(cfg), counts.ctypes.data_as(ctypes.c_void_p), _p(offsets),
                                          _p(padded_offsets), _p(z_codes), _p(z_sf), _p(z_global), _p(w1), _p(w2),
                                          _p(a_global), _p(gate), _p(dy), int(seed), int(rht_signs), _p(dz),
                                          _p(dgate), _p(dw1), _p(dw2), _p(ws), ws.numel(), _stream(stream)),
           "lmoe_expert_backward_nvfp4")
    return ws


def grads(**kw) -> Grads:
    """lmoe_grads from device tensors (missing ones NULL)."""
    return Grads(**{k: _p(v) for k, v in kw.items()})


def backward_nvfp4(cfg: Config, w: Weights, x, dout, a_global, seed, rht_signs, g: Grads, ws=None, stream=None):
    """lmoe_backward_nvfp4: the layer's gradients, routed experts under the
    NVFP4 training recipe (see the header). Allocates the workspace when none
    is given; returns it (its error word holds device errors)."""
    if ws is None:
        import torch
        ws = torch.zeros(int(lib.lmoe_backward_nvfp4_workspace(ctypes.byref(cfg))), dtype=torch.uint8, device="cuda")
    _check(lib.lmoe_backward_nvfp4(ctypes.byref(cfg), ctypes.byref(w), _p(x), _p(dout), _p(a_global), int(seed),
                                   int(rht_signs), ctypes.byref(g), _p(ws), ws.numel(), _stream(stream)),
           "lmoe_backward_nvfp4")
    return ws


def ep_plan(G: int, rank: int, counts):
    """lmoe_ep_plan on host arrays: counts [G][N] int32 (numpy). Returns a dict
    of numpy int32 arrays (send/recv counts and offsets, the local
    expert-grouped layout, the (source, local expert) blocks)."""
    import numpy as np
    counts = np.ascontiguousarray(counts, dtype=np.int32)
    N = counts.shape[1]
    out = {k: np.zeros(G, dtype=np.int32) for k in ("send_counts", "send_offsets", "recv_counts", "recv_offsets")}
    fe, nl = ctypes.c_int32(0), ctypes.c_int32(0)
    lo = np.zeros(N + 1, dtype=np.int32)
    lpo = np.zeros(N + 1, dtype=np.int32)
    bs = np.zeros(G * N, dtype=np.int32)
    bd = np.zeros(G * N, dtype=np.int32)
    br = np.zeros(G * N, dtype=np.int32)
    ptr = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    _check(lib.lmoe_ep_plan(G, rank, N, ptr(counts), ptr(out["send_counts"]), ptr(out["send_offsets"]),
                            ptr(out["recv_counts"]), ptr(out["recv_offsets"]), ctypes.byref(fe), ctypes.byref(nl),
                            ptr(lo), ptr(lpo), ptr(bs), ptr(bd), ptr(br)), "lmoe_ep_plan")
    n = nl.value
    out.update(first_expert=fe.value, local_experts=n, local_offsets=lo[:n + 1], local_padded_offsets=lpo[:n + 1],
               block_src=bs[:G * n], block_dst=bd[:G * n], block_rows=br[:G * n])
    return out


def ep_reorder(x, out, row_bytes, src_rows, dst_rows, row_prefix, total_rows, stream=None):
    """lmoe_ep_reorder: copy row blocks (device tensors; row_prefix int64)."""
    _check(lib.lmoe_ep_reorder(_p(x), _p(out), int(row_bytes), int(src_rows.numel()), _p(src_rows), _p(dst_rows),
                               _p(row_prefix), int(total_rows), _stream(stream)), "lmoe_ep_reorder")


def ep_slot_bases(G: int, rank: int, counts):
    """lmoe_ep_slot_bases on host arrays: counts [G][N] int32 (numpy) ->
    (expert_owner [N], dst_base [N]) numpy int32 arrays for this rank."""
    import numpy as np
    counts = np.ascontiguousarray(counts, dtype=np.int32)
    N = counts.shape[1]
    owner = np.zeros(N, dtype=np.int32)
    base = np.zeros(N, dtype=np.int32)
    ptr = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    _check(lib.lmoe_ep_slot_bases(G, rank, N, ptr(counts), ptr(owner), ptr(base)), "lmoe_ep_slot_bases")
    return owner, base


def ep_dispatch(T, K, N, G, rows, row_bytes, topk_idx, inv_perm, offsets, expert_owner, dst_base, peer_rows,
                peer_rows_cap, topk_w=None, peer_gates=None, err_word=None, stream=None):
    """lmoe_ep_dispatch: this rank's token rows (and gates) stored at their
    slots' rows in the owners' buffers. peer_rows / peer_gates: int64 device
    tensors of the G buffers' addresses."""
    _check(lib.lmoe_ep_dispatch(int(T), int(K), int(N), int(G), _p(rows), int(row_bytes), _p(topk_idx), _p(inv_perm),
                                _p(offsets), _p(expert_owner), _p(dst_base), _p(peer_rows), int(peer_rows_cap),
                                _p(topk_w), _p(peer_gates), _p(err_word), _stream(stream)), "lmoe_ep_dispatch")


def ep_combine(T, K, N, G, l, peer_y, peer_rows_cap, topk_idx, inv_perm, offsets, expert_owner, dst_base, c,
               err_word=None, stream=None):
    """lmoe_ep_combine: c[t] = the k-ordered fp32 sum of the owners' expert
    rows of the token's slots (peer_y: int64 device tensor of addresses)."""
    _check(lib.lmoe_ep_combine(int(T), int(K), int(N), int(G), int(l), _p(peer_y), int(peer_rows_cap),
                               _p(topk_idx), _p(inv_perm), _p(offsets), _p(expert_owner), _p(dst_base), _p(c),
                               _p(err_word), _stream(stream)), "lmoe_ep_combine")


def selftest_wait_timeout(ws, limit_cycles: int, stream=None):
    """lmoe_selftest_wait_timeout: a bounded device wait that runs out."""
    _check(lib.lmoe_selftest_wait_timeout(_p(ws), ws.numel(), int(limit_cycles), _stream(stream)),
           "lmoe_selftest_wait_timeout")


def read_device_error(ws, stream=None):
    """Synchronise, return (status, info) of the workspace's error word and clear it."""
    info = ctypes.c_uint32(0)
    st = lib.lmoe_read_device_error(_p(ws), _stream(stream), ctypes.byref(info))
    return int(st), int(info.value)
