"""The C-ABI library loads on a host without a GPU, exports every function
include/lmoe.h declares, and rejects invalid arguments on the host before
launching anything (no compute calls here)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _ensure_built():
    import importlib.util
    spec = importlib.util.spec_from_file_location("lmoe_build", os.path.join(ROOT, "latentmoe_fwd_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()


_ensure_built()
import latentmoe_fwd_b200 as L  # noqa: E402


def _declared():
    src = open(os.path.join(ROOT, "include", "lmoe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(lmoe_\w+)\s*\(", src)))


def test_header_declares_the_entry_points():
    names = _declared()
    for want in ("lmoe_route", "lmoe_permute", "lmoe_expert_ffn", "lmoe_combine", "lmoe_forward",
                 "lmoe_nvfp4_quantize", "lmoe_workspace_size", "lmoe_read_device_error",
                 "lmoe_status_string"):
        assert want in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(L.LIB_PATH)
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_wraps_every_export():
    assert set(L.EXPORTS) <= set(_declared())


def test_status_strings():
    assert L.status_string(L.OK) == "ok"
    assert "workspace" in L.status_string(L.ERR_WORKSPACE)


def test_workspace_sizes_and_padded_rows():
    cfg = L.config(T=16384, d=8192, l=2048, N=512, K=22, m=1024)
    assert L.padded_rows(cfg) == ((16384 * 22 + 127 * 512 + 127) // 128) * 128
    fwd = L.workspace_size(cfg, L.OP_FORWARD)
    assert fwd > 3 * 16384 * 22 * 2048 * 2          # z_perm, y and a at least
    assert L.workspace_size(cfg, L.OP_COMBINE) == 0
    assert 0 < L.workspace_size(cfg, L.OP_ROUTE) < fwd
    bad = L.config(T=4, d=64, l=64, N=4, K=5, m=64)    # K > N
    assert L.workspace_size(bad, L.OP_FORWARD) == 0
    # the token limit: 2^25 tokens are accepted, one more is not
    assert L.workspace_size(L.config(T=2**25, d=64, l=64, N=8, K=2, m=64), L.OP_FORWARD) > 0
    assert L.workspace_size(L.config(T=2**25 + 1, d=64, l=64, N=8, K=2, m=64), L.OP_FORWARD) == 0


@pytest.mark.parametrize("kw,status", [
    (dict(K=5), L.ERR_INVALID_ARG),               # K > N
    (dict(K=33, N=64), L.ERR_UNSUPPORTED),        # K above the warp-per-token limit
    (dict(d=60), L.ERR_INVALID_ARG),              # rows not a multiple of 16 bytes
    (dict(act=L.F32, expert=L.BF16), L.ERR_UNSUPPORTED),
    (dict(expert=L.NVFP4, l=128), L.ERR_UNSUPPORTED),
    (dict(expert=L.NVFP4, l=256, m=128), L.ERR_UNSUPPORTED),
    (dict(T=-1), L.ERR_INVALID_ARG),
    (dict(T=2**25 + 1), L.ERR_INVALID_ARG),
    (dict(m=0), L.ERR_INVALID_ARG),
    (dict(l=60), L.ERR_INVALID_ARG),
    (dict(identity=True, l=32), L.ERR_INVALID_ARG),
    (dict(n_shared=-1), L.ERR_INVALID_ARG),
    (dict(n_shared=1, m_shared=0), L.ERR_INVALID_ARG),
    (dict(n_shared=1, m_shared=36), L.ERR_INVALID_ARG),
    (dict(n_shared=1, m_shared=40), L.ERR_UNSUPPORTED),   # BF16 shared experts: m_shared % 64
    (dict(N=1032, K=2), L.ERR_UNSUPPORTED),
    (dict(expert=L.F32), L.ERR_UNSUPPORTED),              # BF16 activations, fp32 experts
    (dict(act=L.NVFP4, expert=L.NVFP4), L.ERR_UNSUPPORTED),
])
def test_invalid_configs_rejected_on_host(kw, status):
    base = dict(T=4, d=64, l=64, N=4, K=2, m=64)
    base.update(kw)
    cfg = L.config(**base)
    w = L.weights(w_router=16, w1=16, w2=16, w_down=16, w_up=16)
    st = L.lib.lmoe_forward(ctypes.byref(cfg), ctypes.byref(w), 16, 16, 16, 1 << 40, None)
    assert st == status


def test_null_and_workspace_errors_rejected_on_host():
    cfg = L.config(T=4, d=64, l=32, N=4, K=2, m=64)
    w = L.weights(w_router=16, w1=16, w2=16, w_down=16, w_up=16)
    # workspace too small
    assert L.lib.lmoe_forward(ctypes.byref(cfg), ctypes.byref(w), 16, 16, 16, 8, None) == L.ERR_WORKSPACE
    # missing w_up while not identity
    w2 = L.weights(w_router=16, w1=16, w2=16, w_down=16)
    assert L.lib.lmoe_forward(ctypes.byref(cfg), ctypes.byref(w2), 16, 16, 16, 1 << 40, None) == L.ERR_INVALID_ARG
    # misaligned x
    assert L.lib.lmoe_forward(ctypes.byref(cfg), ctypes.byref(w), 18, 16, 16, 1 << 40, None) == L.ERR_INVALID_ARG
    # route needs outputs
    assert L.lib.lmoe_route(ctypes.byref(cfg), 16, 16, None, None, None, None, None, 16, 1 << 20,
                            None) == L.ERR_INVALID_ARG
    # nvfp4: cols must be a multiple of 16
    assert L.lib.lmoe_nvfp4_quantize(16, L.BF16, 4, 24, None, 16, 16, None, 0, 16, 1 << 20,
                                     None) == L.ERR_INVALID_ARG
    # permute: rows without a destination
    assert L.lib.lmoe_permute(ctypes.byref(cfg), 16, 16, 16, 16, 16, 16, 64, None, None, None, None, None,
                              16, 1 << 20, None) == L.ERR_INVALID_ARG


def test_launch_counter_starts_and_is_monotone():
    a = L.kernel_launch_count()
    b = L.kernel_launch_count()
    assert b >= a >= 0


def test_nvfp4_quantize_layout_flags():
    src = open(os.path.join(ROOT, "include", "lmoe.h")).read()
    assert "#define LMOE_SF_BLOCK_16X16 0x10" in src
    assert L.SF_BLOCK_16X16 == 0x10
    ws = ctypes.create_string_buffer(4096)
    fake = ctypes.c_void_p(4096)   # never dereferenced: the layout is rejected first
    for bad in (2, 3, 0x20, 0x12):
        st = L.lib.lmoe_nvfp4_quantize(fake, 1, 16, 16, None, fake, fake, None, bad, ws, 4096, None)
        assert st == L.ERR_INVALID_ARG


def test_selftest_wait_rejects_bad_arguments_on_host():
    small = ctypes.create_string_buffer(128)
    assert L.lib.lmoe_selftest_wait_timeout(small, 128, 1000, None) == L.ERR_WORKSPACE
    ws = ctypes.create_string_buffer(256)
    assert L.lib.lmoe_selftest_wait_timeout(ws, 256, 0, None) == L.ERR_INVALID_ARG
    assert L.lib.lmoe_selftest_wait_timeout(ws, 256, 5_000_000_000, None) == L.ERR_INVALID_ARG


def test_router_gemm_needs_n_multiple_of_8():
    cfg = L.config(T=4, d=64, l=64, N=4, K=2, m=64)
    w = L.weights(w_router=16, w1=16, w2=16, w_down=16, w_up=16)
    assert L.lib.lmoe_forward(ctypes.byref(cfg), ctypes.byref(w), 16, 16, 16, 1 << 40, None) == L.ERR_UNSUPPORTED
    idx = 16
    assert L.lib.lmoe_route(ctypes.byref(cfg), 16, 16, None, None, idx, idx, None, 16, 1 << 30,
                            None) == L.ERR_UNSUPPORTED


def test_noalloc_permute_host_checks():
    def call(cfg):
        return L.lib.lmoe_permute_noalloc(ctypes.byref(cfg), 16, 16, 16, 16, 16, None, 0, None, None, None,
                                          None, None, None)
    assert call(L.config(T=2**25 + 1, d=8, l=8, N=8, K=2, m=8)) == L.ERR_INVALID_ARG
    assert call(L.config(T=4, d=8, l=8, N=4, K=5, m=8)) == L.ERR_INVALID_ARG          # K > N
    assert call(L.config(T=4, d=8, l=8, N=2048, K=2, m=8)) == L.ERR_UNSUPPORTED
    # beyond the fixed 131072-counter scratch: (ceil(T*K / 8192) + 1) * N counters
    assert call(L.config(T=300000, d=8, l=8, N=1024, K=8, m=8)) == L.ERR_WORKSPACE


def test_documented_host_errors_of_each_entry_point():
    P = ctypes.byref
    cfg = L.config(T=4, d=64, l=32, N=8, K=2, m=64)
    w = L.weights(w_router=16, w1=16, w2=16, w_down=16, w_up=16)
    big = 1 << 40
    # expert FFN: missing weights, unaligned output, NVFP4 without scales
    assert L.lib.lmoe_expert_ffn(P(cfg), P(L.weights(w1=16)), 16, None, None, 16, 16, None, 16, 16, big,
                                 None) == L.ERR_INVALID_ARG
    assert L.lib.lmoe_expert_ffn(P(cfg), P(w), 16, None, None, 16, 16, None, 24, 16, big, None) == L.ERR_INVALID_ARG
    assert L.lib.lmoe_expert_ffn(P(cfg), P(w), 16, None, None, 16, 16, None, 16, 16, 8, None) == L.ERR_WORKSPACE
    cfg4 = L.config(T=4, d=256, l=256, N=8, K=2, m=256, expert=L.NVFP4)
    assert L.lib.lmoe_expert_ffn(P(cfg4), P(w), 16, 16, 16, 16, 16, None, 16, 16, big, None) == L.ERR_INVALID_ARG
    # combine: NULL or unaligned buffers
    assert L.lib.lmoe_combine(P(cfg), None, 16, 16, 16, 16, None, 16, None) == L.ERR_INVALID_ARG
    assert L.lib.lmoe_combine(P(cfg), 16, 16, 16, 16, 16, None, 40, None) == L.ERR_INVALID_ARG
    # forward: projections given with the identity flag; missing shared weights
    ident = L.config(T=4, d=64, l=64, N=8, K=2, m=64, identity=True)
    assert L.lib.lmoe_forward(P(ident), P(w), 16, 16, 16, big, None) == L.ERR_INVALID_ARG
    shared = L.config(T=4, d=64, l=32, N=8, K=2, m=64, n_shared=1, m_shared=64)
    assert L.lib.lmoe_forward(P(shared), P(w), 16, 16, 16, big, None) == L.ERR_INVALID_ARG
    # reading the error word needs a workspace
    info = ctypes.c_uint32(0)
    assert L.lib.lmoe_read_device_error(None, None, ctypes.byref(info)) == L.ERR_INVALID_ARG


def test_fp8_shared_config_checks():
    """LMOE_FLAG_SHARED_FP8: m_shared must be a multiple of 128 and there must
    be shared experts (host-side checks; no GPU needed)."""
    base = dict(T=64, d=512, l=256, N=8, K=2, m=256, shared_fp8=True)
    assert L.workspace_size(L.config(**base, n_shared=2, m_shared=64), L.OP_FORWARD) == 0
    assert L.workspace_size(L.config(**base, n_shared=0, m_shared=0), L.OP_FORWARD) == 0
    assert L.workspace_size(L.config(**base, n_shared=2, m_shared=128), L.OP_FORWARD) > 0
    assert L.workspace_size(L.config(T=100, d=64, l=64, N=1, K=1, m=64), L.OP_FP8_QUANTIZE) > 0


def test_fp8_quantize_host_errors():
    dummy = 256   # a fake aligned address; nothing is launched on these errors
    with pytest.raises(L.LmoeError) as e:
        L.fp8_quantize(dummy, L.BF16, 4, 24, None, dummy, None, stream=0)   # cols % 16
    assert e.value.status == L.ERR_INVALID_ARG
    with pytest.raises(L.LmoeError) as e:
        L.fp8_quantize(dummy, L.BF16, 4, 32, None, dummy, None, stream=0)   # amax scale needs a workspace
    assert e.value.status == L.ERR_WORKSPACE


def test_transpose_and_ep_kernels_host_errors():
    # argument checks that return before any device work
    assert L.lib.lmoe_nvfp4_transpose_2d(16, 16, 1, 128, 128, None, 16, None) == L.ERR_INVALID_ARG
    assert L.lib.lmoe_nvfp4_transpose_2d(16, 16, 1, 100, 128, 16, 16, None) == L.ERR_UNSUPPORTED   # rows % 128
    assert L.lib.lmoe_nvfp4_transpose_2d(16, 16, 1, 128, 128, 24, 16, None) == L.ERR_INVALID_ARG   # unaligned
    assert L.lib.lmoe_nvfp4_transpose_2d(None, None, 0, 128, 128, None, None, None) == L.OK        # nothing to do
    assert L.lib.lmoe_ep_dispatch(4, 0, 8, 2, 16, 32, 16, 16, 16, 16, 16, 16, 64, None, None, None,
                                  None) == L.ERR_INVALID_ARG                                        # K = 0
    assert L.lib.lmoe_ep_dispatch(4, 2, 8, 2, 16, 24, 16, 16, 16, 16, 16, 16, 64, None, None, None,
                                  None) == L.ERR_INVALID_ARG                                        # row bytes % 16
    assert L.lib.lmoe_ep_dispatch(4, 2, 8, 2, 16, 32, 16, 16, 16, 16, 16, 16, 64, 16, None, None,
                                  None) == L.ERR_INVALID_ARG                                        # gates, no buffers
    assert L.lib.lmoe_ep_dispatch(0, 2, 8, 2, None, 0, None, None, None, None, None, None, 0, None, None, None,
                                  None) == L.OK                                                     # no tokens
    assert L.lib.lmoe_ep_combine(4, 2, 8, 2, 36, 16, 64, 16, 16, 16, 16, 16, 16, None,
                                 None) == L.ERR_INVALID_ARG                                         # l % 8
    assert L.lib.lmoe_ep_combine(4, 2, 8, 2, 64, 16, 64, 16, 16, 16, 16, 16, 24, None,
                                 None) == L.ERR_INVALID_ARG                                         # unaligned c


def test_binding_rejects_host_tensors():
    # a torch tensor in host memory never reaches the library as a pointer
    import torch
    cfg = L.config(T=4, d=64, l=32, N=8, K=2, m=64)
    x = torch.zeros((4, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        L.forward(cfg, L.weights(w_router=16, w1=16, w2=16, w_down=16, w_up=16), x, 16, x, stream=0)
    with pytest.raises(ValueError):
        L.weights(w_router=x)
    with pytest.raises(ValueError):
        L.grads(dx=x)
    assert L._p(None) is None and L._p(4096) == 4096
