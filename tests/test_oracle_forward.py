"""Pins for the oracle's whole-layer forward.

Structure (greeksharifa page on the Nemotron 3 whitepaper, section 2.2
"LatentMoE"; notes.yuuk.io page, section 2 "LatentMoE"): project x from d down
to l, run the routed experts in l, combine, project back to d; router and
shared experts read the d-dim x. Pinned here by:

* the dense all-experts formula out_t = W_up sum_e G[t,e] FFN_e(W_dn x_t)
  + sum_s FFN_s(x_t), with a T x N gate matrix in place of dispatch;
* invariant (c): l = d, identity projections, no shared experts equals an
  independently coded standard MoE;
* the concatenation identity of shared experts, K = 1, linearity in W_up;
* a per-token scalar-loop rendition of the BF16 rounding points;
* seeded-generator determinism.
"""
from dataclasses import replace

import numpy as np
import pytest

import lmoe_inputs as LI
from oracle import lmoe_oracle as O


def _tiny(dtype="bf16", identity=False, n_shared=0, **kw):
    base = dict(name="t", T=9, d=32, l=16, N=6, K=2, m=24, n_shared=n_shared,
                m_shared=16 if n_shared else 0, dtype=dtype, identity=identity)
    if identity:
        base["l"] = base["d"]
    base.update(kw)
    return LI.Workload(**base)


def _f64_inputs(wl, inp):
    st = "f32" if wl.dtype == "f32" else "bf16"
    return {k: (O.to_f64(v, st) if isinstance(v, np.ndarray) and k != "router_bias" else v)
            for k, v in inp.items()}


def _ffn(w1, w2, v):
    return w2 @ O.sq_relu(w1 @ v)


def _dense_formula(wl, inp):
    f = _f64_inputs(wl, inp)
    x = f["x"]
    logits = x @ f["w_router"].T
    if inp["router_bias"] is not None:
        logits = logits + inp["router_bias"].astype(np.float64)
    idx, gates = O.route_topk(logits, wl.K)
    G = np.zeros((wl.T, wl.N))
    for t in range(wl.T):
        G[t, idx[t]] = gates[t]
    out = np.zeros((wl.T, wl.d))
    for t in range(wl.T):
        z = x[t] if wl.identity else f["w_down"] @ x[t]
        c = sum(G[t, e] * _ffn(f["w1"][e], f["w2"][e], z) for e in range(wl.N))
        o = c if wl.identity else f["w_up"] @ c
        for s in range(wl.n_shared):
            o = o + _ffn(f["ws1"][s], f["ws2"][s], x[t])
        out[t] = o
    return out


@pytest.mark.parametrize("identity,n_shared", [(False, 0), (False, 2), (True, 0), (True, 2)])
def test_dispatch_forward_equals_dense_formula(identity, n_shared):
    wl = _tiny(identity=identity, n_shared=n_shared)
    inp = LI.make_inputs(wl)
    got = O.forward(wl, inp, precision="f64")["out"]
    ref = _dense_formula(wl, inp)
    assert np.max(np.abs(got - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref)))


def test_zipf_bias_enters_selection_and_gates():
    wl = _tiny(zipf_bias=True, T=12, N=8, K=3)
    inp = LI.make_inputs(wl)
    assert inp["router_bias"] is not None
    got = O.forward(wl, inp, precision="f64")["out"]
    ref = _dense_formula(wl, inp)
    assert np.max(np.abs(got - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref)))


def test_identity_layer_equals_standard_moe():
    """Invariant (c), with a standard MoE coded independently per token."""
    wl = _tiny(identity=True, T=11, N=5, K=2)
    inp = LI.make_inputs(wl)
    f = _f64_inputs(wl, inp)
    got = O.forward(wl, inp, precision="f64")["out"]
    for t in range(wl.T):
        x = f["x"][t]
        s = np.array([x @ f["w_router"][e] for e in range(wl.N)])
        chosen = sorted(range(wl.N), key=lambda e: (-s[e], e))[:wl.K]
        w = np.exp(s[chosen] - s[chosen].max())
        w /= w.sum()
        ref = np.zeros(wl.d)
        for g, e in zip(w, chosen):
            h = np.maximum(f["w1"][e] @ x, 0.0) ** 2
            ref += g * (f["w2"][e] @ h)
        assert np.max(np.abs(got[t] - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref)))


def test_two_shared_experts_equal_one_of_double_width():
    wl = _tiny(n_shared=2, T=7)
    inp = LI.make_inputs(wl)
    two = O.forward(wl, inp, precision="f64")["out"]
    wl1 = replace(wl, n_shared=1, m_shared=2 * wl.m_shared)
    inp1 = dict(inp)
    inp1["ws1"] = np.concatenate([inp["ws1"][0], inp["ws1"][1]], axis=0)[None]
    inp1["ws2"] = np.concatenate([inp["ws2"][0], inp["ws2"][1]], axis=1)[None]
    one = O.forward(wl1, inp1, precision="f64")["out"]
    assert np.max(np.abs(two - one)) <= 1e-12 * np.max(np.abs(two))


def test_k1_is_single_expert_ffn():
    wl = _tiny(K=1, T=8)
    inp = LI.make_inputs(wl)
    f = _f64_inputs(wl, inp)
    r = O.forward(wl, inp, precision="f64")
    for t in range(wl.T):
        e = r["idx"][t, 0]
        ref = f["w_up"] @ _ffn(f["w1"][e], f["w2"][e], f["w_down"] @ f["x"][t])
        assert np.max(np.abs(r["out"][t] - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref)))


def test_linear_in_w_up():
    wl = _tiny(T=6)
    inp = LI.make_inputs(wl)
    base = O.forward(wl, inp, precision="f64")["out"]
    inp2 = dict(inp)
    w_up = O.from_bf16_bits(inp["w_up"]) * 2.0      # exact doubling in BF16
    inp2["w_up"] = LI.bf16_bits(w_up)
    doubled = O.forward(wl, inp2, precision="f64")["out"]
    assert np.max(np.abs(doubled - 2 * base)) <= 1e-12 * np.max(np.abs(base))


def _bf16_scalar_loops(wl, inp):
    """The BF16 layer, token by token with scalar dot products, rounding at z,
    a, y (after the gate), c and out, and at the shared experts' hidden."""
    f = _f64_inputs(wl, inp)
    R = O.round_bf16
    out = np.zeros((wl.T, wl.d))
    for t in range(wl.T):
        x = f["x"][t]
        s = [float(np.dot(x, f["w_router"][e])) for e in range(wl.N)]
        chosen = sorted(range(wl.N), key=lambda e: (-s[e], e))[:wl.K]
        ex = [np.exp(s[e] - max(s)) for e in chosen]
        gates = [v / sum(ex) for v in ex]
        z = [R(float(np.dot(f["w_down"][i], x))) for i in range(wl.l)]
        c = [0.0] * wl.l
        for g, e in zip(gates, chosen):
            a = [R(max(float(np.dot(f["w1"][e][j], z)), 0.0) ** 2) for j in range(wl.m)]
            for i in range(wl.l):
                c[i] += R(g * float(np.dot(f["w2"][e][i], a)))
        c = [R(v) for v in c]
        for j in range(wl.d):
            v = float(np.dot(f["w_up"][j], c))
            for sh in range(wl.n_shared):
                hs = [R(max(float(np.dot(f["ws1"][sh][q], x)), 0.0) ** 2) for q in range(wl.m_shared)]
                v += float(np.dot(f["ws2"][sh][j], hs))
            out[t, j] = R(v)
    return out


def test_bf16_rounding_points_match_scalar_loops():
    wl = _tiny(T=5, n_shared=1)
    inp = LI.make_inputs(wl)
    got = O.forward(wl, inp)["out"]
    ref = _bf16_scalar_loops(wl, inp)
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 7)
    assert np.all(np.abs(got - ref) <= ulp)                 # at most one BF16 step
    assert np.mean(got == ref) >= 0.97                      # and almost always identical


def test_bf16_rounding_differs_from_unrounded():
    wl = _tiny(T=5)
    inp = LI.make_inputs(wl)
    r = O.forward(wl, inp)["out"]
    assert np.array_equal(r, O.round_bf16(r))               # out lies on the BF16 grid
    r64 = O.forward(wl, inp, precision="f64")["out"]
    assert not np.array_equal(r, r64)


def test_token_subset_equals_full_rows():
    wl = _tiny(T=10)
    inp = LI.make_inputs(wl)
    full = O.forward(wl, inp)["out"]
    sub = O.forward(wl, inp, tokens=[7, 2, 9])["out"]
    assert np.array_equal(sub, full[[7, 2, 9]])


def test_f32_workload_rounds_to_fp32():
    wl = _tiny(dtype="f32", T=6)
    inp = LI.make_inputs(wl)
    assert inp["x"].dtype == np.float32
    r = O.forward(wl, inp)["out"]
    assert np.array_equal(r, O.round_f32(r))


def test_nvfp4_forward_fake_quantises_z_and_a():
    wl = _tiny(dtype="nvfp4", T=8, d=64, l=32, m=48, outliers=True)
    inp = LI.make_inputs(wl)
    r = O.forward(wl, inp)
    z = r["z"]
    zq, _ = O.nvfp4_fake_quant(z, r["z_global_scale"])
    assert np.array_equal(z, zq)                            # z already on its NVFP4 grid
    a = r["a"]
    aq, _ = O.nvfp4_fake_quant(a, inp["a_global_scale"])
    assert np.array_equal(a, aq)
    # and it stays close to the BF16 layer (a quantisation, not a different layer)
    rb = O.forward(replace(wl, dtype="bf16"), inp)["out"]
    rel = np.sqrt(np.mean((r["out"] - rb) ** 2) / np.mean(rb ** 2))
    assert rel < 0.3


def test_generator_is_deterministic_and_thread_independent():
    wl = _tiny(zipf_bias=True, outliers=True, n_shared=2)
    a = LI.make_inputs(wl, threads=1)
    b = LI.make_inputs(wl, threads=4)
    for k in a:
        if isinstance(a[k], np.ndarray):
            assert np.array_equal(a[k], b[k]), k
    n_out = int(round(0.001 * wl.T * wl.d))
    assert n_out >= 0


def test_generator_distributions():
    wl = LI.Workload("g", T=256, d=512, l=128, N=8, K=2, m=64)
    inp = LI.make_inputs(wl)
    x = O.from_bf16_bits(inp["x"])
    assert abs(x.std() - 1.0) < 0.02
    w1 = O.from_bf16_bits(inp["w1"])
    assert abs(w1.std() * np.sqrt(wl.l) - 1.0) < 0.02
    w2 = O.from_bf16_bits(inp["w2"])
    assert abs(w2.std() * np.sqrt(wl.m) - 1.0) < 0.02


def test_outlier_count():
    wl = LI.Workload("o", T=100, d=200, l=32, N=4, K=2, m=32, dtype="nvfp4", outliers=True)
    inp = LI.make_inputs(wl)
    x = O.from_bf16_bits(inp["x"])
    assert np.sum(np.abs(x) > 12) <= int(round(0.001 * wl.T * wl.d))
    assert np.sum(np.abs(x) > 12) >= 1


def test_correctly_rounded_bf16_output_can_exceed_two_percent_of_rms():
    """Why the BF16 parity bar is applied beyond half a BF16 step: the exact
    layer output rounded to BF16 (the best any BF16 output can do) already
    misses the exact value by more than 2e-2 * RMS on this seeded case."""
    wl = LI.reduced("ultra_zipf", T=900, d=1024, l=512, N=32, K=6, m=512)
    inp = LI.make_inputs(wl)
    r = O.forward(wl, inp)
    rms = np.sqrt(np.mean(r["out"] ** 2))
    representation = np.max(np.abs(O.round_bf16(r["out_unrounded"]) - r["out_unrounded"])) / rms
    assert representation > 2e-2
    _, e = np.frexp(np.abs(r["out"]))
    half_step = np.ldexp(1.0, np.maximum(e - 1, -126) - 7) / 2
    assert np.all(np.abs(O.round_bf16(r["out_unrounded"]) - r["out_unrounded"]) <= half_step)


def test_nvfp4_z_rows_override_and_weight_cache_are_transparent():
    wl = _tiny(dtype="nvfp4", T=6, d=64, l=32, m=48, outliers=True)
    inp = LI.make_inputs(wl)
    base = O.forward(wl, inp)
    x = O.from_bf16_bits(inp["x"])
    z_full = O.round_bf16(x @ O.from_bf16_bits(inp["w_down"]).T)
    W = O.weights_view(wl, inp, cache=True)
    same = O.forward(wl, inp, tokens=[1, 4], z_rows=z_full[[1, 4]], weights=W)
    assert np.array_equal(same["out"], base["out"][[1, 4]])
    again = O.forward(wl, inp, tokens=[1, 4], weights=W)      # cached quantised experts
    assert np.array_equal(again["out"], base["out"][[1, 4]])
    # a different z row changes that token only through its own quantised latent
    alt = z_full[[1]].copy()
    alt[0, 0] = -alt[0, 0] + 1.0
    moved = O.forward(wl, inp, tokens=[1], z_rows=alt, weights=W)
    assert not np.array_equal(moved["out"], base["out"][[1]])
