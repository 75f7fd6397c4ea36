"""Throughput of the LatentMoE layer forward on B200 (one JSON line on stdout).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one whole layer forward (router, top-K, down-projection,
permutation, expert GEMMs, combine, up-projection and shared experts) over
one batch of T synthetic tokens, through the library's C ABI.

* value:   tokens/s of all ranks with inputs already resident in HBM, timed
           with CUDA events over exactly K steps (max over ranks).
* e2e:     the same metric with every step's input copied from pinned host
           memory and its output copied back to pinned host memory, the copies
           on their own streams (double-buffered) overlapping the forwards.
* roofline: the grouped expert GEMM launches (the dominant kernel), timed
           with CUDA events recorded by the library at its stage boundaries
           on the launch stream (a pass of K forwards right after the timed
           region). Their algorithmic work is the layer's own: the used
           experts' weights once (bytes) and 2*T*K*l*m*2 (flops); the binding
           roof is the slower of the two at the measured burst peaks.
* cpu_baseline: the fp64 CPU oracle on a bounded sample of the same workload
           (rank 0, N = 1 only).

--impl reference times the oracle itself (the reference arm of this path) on
the host cores, on bounded samples of the same workload.

With N > 1 (torchrun) every rank runs an independent replica on its own batch
(no data-path collective; weak scaling); the process group only carries the
barrier and the max over ranks.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import lmoe_inputs as LI  # noqa: E402

METRIC = "LatentMoE layer fwd tokens/s on 1 B200; % of HBM (decode) or tensor (prefill) peak"
DEFAULT_WORKLOAD = "ultra_zipf"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------------------
# clocks sampled during the timed region
# --------------------------------------------------------------------------
REASON_FIELDS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")


class ClockSampler:
    def __init__(self, device_index: int):
        q = ("index,clocks.sm,clocks.max.sm,power.draw,"
             + ",".join(f"clocks_event_reasons.{r}" for r in REASON_FIELDS))
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits", "-lms", "20",
                 "-i", str(device_index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], None, set()
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 4 + len(REASON_FIELDS):
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for name, v in zip(REASON_FIELDS, parts[4:]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------------
# algorithmic work of the dominant kernel (the two grouped expert GEMMs)
# --------------------------------------------------------------------------
def expert_gemm_work(wl, counts: np.ndarray):
    """Algorithmic work of expert GEMM 1 + GEMM 2 (the two grouped launches)
    for one forward, by the layer's definition rather than this design's
    data movement.

    bytes: W1_e and W2_e of every expert that received at least one row, each
      read once, in the workload's weight format (NVFP4: 0.5 byte per element
      plus one E4M3 scale per 16), plus the shared experts' Ws1 and Ws2 where
      their two layers run in the same launches.
    flops: 2 * (T*K) * l * m * 2 (+ 2 * T * d * S * m_s * 2 with the shared
      layers).
    traffic_model: the activation rows the two launches read and write in this
      design (gathered z rows in, a out and back in, y out; with the shared
      layers x in, hs out and back in, ys out). They are intermediates the
      design materialises, reported beside the algorithmic bytes, not in them.
    Returns (bytes, flops, experts used, traffic_model bytes).
    """
    rows = int(counts.sum())
    used = int(np.count_nonzero(counts))
    if wl.dtype == "nvfp4":
        q = 0.5 + 1.0 / 16
        wbytes = used * 2 * wl.m * wl.l * q
        abytes = rows * (wl.l + wl.m) * q + rows * (wl.m * q + wl.l * 2)
    else:
        eb = 4 if wl.dtype == "f32" else 2
        wbytes = used * 2 * wl.m * wl.l * eb
        abytes = rows * (wl.l + wl.m) * eb * 2
    flops = 2.0 * rows * wl.l * wl.m * 2
    if wl.n_shared and shared_fused(wl):
        sm = wl.n_shared * wl.m_shared
        wbytes += 2 * sm * wl.d * 2
        abytes += wl.T * wl.d * 2 * 2 + wl.T * sm * 2 * 2
        flops += 2.0 * wl.T * wl.d * sm * 2
    return wbytes, flops, used, abytes


def pair_tiles(wl) -> bool:
    """Grouped BF16 expert GEMMs run on CTA pairs (T > 64, >= 64 rows per expert)."""
    return wl.dtype == "bf16" and wl.T > 64 and wl.T * wl.K >= 64 * wl.N


def shared_fused(wl) -> bool:
    """The shared experts' layers ride along in the CTA-pair expert-GEMM launches."""
    return bool(wl.n_shared) and pair_tiles(wl)


GEMM_SOURCES = ("gemm_tc.cuh", "gemm_tc2.cuh", "gemm_fp4.cuh", "lmoe_device.cuh")


def gemm_source_sha() -> str:
    """sha256 prefix over the expert-GEMM kernel sources (traffic figures
    taken with ncu stay valid only while these are unchanged)."""
    h = hashlib.sha256()
    for name in GEMM_SOURCES:
        with open(os.path.join(ROOT, "latentmoe_fwd_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def expert_gemm_kernel(wl) -> str:
    """The kernel that runs the grouped expert GEMMs of this workload."""
    if wl.dtype == "nvfp4":
        return "fp4_gemm_kernel (grouped NVFP4 expert GEMM 1 + GEMM 2, 2 launches per step)"
    if wl.dtype == "f32":
        return "simt_gemm_kernel (fp32 layer)"
    if pair_tiles(wl):
        extra = " with the shared experts' hidden and output layers" if shared_fused(wl) else ""
        return f"tc2_gemm_kernel (CTA-pair grouped expert GEMM 1 + GEMM 2{extra}, 2 launches per step)"
    return "tc_gemm_kernel (grouped expert GEMM 1 + GEMM 2, 2 launches per step)"


def traffic_record(workload: str):
    """DRAM traffic per expert-GEMM launch pair from a committed ncu capture,
    valid only while the GEMM source is unchanged."""
    p = os.path.join(ROOT, "profiles", "expert_gemm_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    h = gemm_source_sha()
    entry = rec.get(workload)
    if not entry or entry.get("gemm_source_sha") != h:
        return None
    return entry.get("traffic_bytes_per_forward")


def quantize_experts(L, w):
    """NVFP4 copies of expert weights [N][rows][cols] through lmoe_nvfp4_quantize:
    packed codes, MMA-tiled block scales and one global scale per expert matrix."""
    import torch
    N, rows, cols = w.shape
    codes = torch.empty((N, rows, cols // 2), dtype=torch.uint8, device="cuda")
    sf = torch.empty((N, rows * cols // 16), dtype=torch.uint8, device="cuda")
    gs = torch.empty(N, dtype=torch.float32, device="cuda")
    ws = L.workspace(L.config(T=rows, d=cols, l=cols, N=1, K=1, m=cols), L.OP_NVFP4_QUANTIZE)
    for e in range(N):
        L.nvfp4_quantize(w[e], L.BF16, rows, cols, None, codes[e], sf[e], gs[e:e + 1], L.SF_MMA_TILED, ws)
    st, info = L.read_device_error(ws)
    if st != L.OK:
        raise RuntimeError(f"weight quantisation failed: {L.status_string(st)}")
    return codes, sf, gs


def quantizer_rates(L, w, hbm_gbs):
    """lmoe_nvfp4_quantize over all experts' W1 as one [N*rows, cols] matrix
    (current amax, MMA-tiled scales), with 1 x 16 and with 16 x 16 scale
    blocks: ms per call and the rate on its algorithmic bytes (the amax pass
    reads the input, the encode pass reads it again and writes codes and
    scales: 2 + 2 + 0.5625 bytes per element)."""
    import torch
    N, rows, cols = w.shape
    R = N * rows
    flat = w.reshape(R, cols)
    codes = torch.empty((R, cols // 2), dtype=torch.uint8, device="cuda")
    sf = torch.empty((((R + 127) // 128) * 128 * (cols // 16),), dtype=torch.uint8, device="cuda")
    g = torch.empty(1, dtype=torch.float32, device="cuda")
    ws = L.workspace(L.config(T=R, d=cols, l=cols, N=1, K=1, m=cols), L.OP_NVFP4_QUANTIZE)
    alg = R * cols * (2 + 2 + 0.5625)
    out = {"rows": R, "cols": cols, "algorithmic_bytes": alg}
    for name, layout in (("1x16", L.SF_MMA_TILED), ("16x16", L.SF_MMA_TILED | L.SF_BLOCK_16X16)):
        L.nvfp4_quantize(flat, L.BF16, R, cols, None, codes, sf, g, layout, ws)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 5
        a.record()
        for _ in range(reps):
            L.nvfp4_quantize(flat, L.BF16, R, cols, None, codes, sf, g, layout, ws)
        b.record()
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / reps
        gbs = alg / (ms / 1000.0) / 1e9
        out[name] = {"ms": ms, "achieved_gbs": gbs, "frac_of_hbm": gbs / hbm_gbs}
    st, info = L.read_device_error(ws)
    if st != L.OK:
        raise RuntimeError(f"quantiser measurement failed: {L.status_string(st)}")
    return out


def roofline(wl, alg_bytes, alg_flops, gemm_ms, peaks, peak_src):
    """Roofline of the expert-GEMM launches against the burst peaks (the
    launches are timed inside millisecond steps, not seconds-long loops).

    The binding roof is the slower of bytes / HBM copy bandwidth and flops /
    dense tensor peak (BF16 burst; NVFP4: 4 x the BF16 burst, the nominal
    9 : 2.25 dense ratio). achieved = algorithmic work / measured launch time,
    frac = achieved / peak. The sustained tensor peak is given beside it."""
    if wl.dtype == "f32":
        return {"bound": "launch", "achieved": None, "peak": None, "unit": None, "frac": None, "traffic": None,
                "algorithmic_bytes": alg_bytes, "algorithmic_flops": alg_flops, "kernel_ms_per_step": gemm_ms}
    ratio = 4.0 if wl.dtype == "nvfp4" else 1.0
    tc_peak = peaks["bf16_tflops"] * ratio
    tc_sust = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]) * ratio
    t_hbm = alg_bytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = alg_flops / (tc_peak * 1e12)
    src = "measured (MEASURED_PEAKS.json)" if peak_src == "measured" else "fallback"
    tc_kind = "bf16_tflops x 4 (nominal FP4 : BF16 dense ratio)" if ratio > 1 else "bf16_tflops"
    if t_hbm >= t_tc:
        ach = alg_bytes / (gemm_ms / 1000.0) / 1e9
        r = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
             "frac": ach / peaks["hbm_gbs"], "peak_kind": "hbm_gbs"}
    else:
        ach = alg_flops / (gemm_ms / 1000.0) / 1e12
        r = {"bound": "tensor", "achieved": ach, "peak": tc_peak, "unit": "TFLOP/s", "frac": ach / tc_peak,
             "peak_kind": tc_kind, "peak_sustained": tc_sust, "frac_of_sustained": ach / tc_sust}
    r.update({"algorithmic_bytes": alg_bytes, "algorithmic_flops": alg_flops, "kernel_ms_per_step": gemm_ms,
              "time_at_hbm_peak_ms": t_hbm * 1e3, "time_at_tensor_peak_ms": t_tc * 1e3, "peak_source": src})
    return r


# --------------------------------------------------------------------------
# the CPU oracle, timed (bounded sample)
# --------------------------------------------------------------------------
def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return len(os.sched_getaffinity(0))


def oracle_tokens_per_s(wl, inp, n_tokens: int, seed: int = 0):
    from oracle import lmoe_oracle as O
    rng = np.random.default_rng(seed)
    toks = np.sort(rng.choice(wl.T, size=min(n_tokens, wl.T), replace=False))
    t0 = time.perf_counter()
    O.forward(wl, inp, tokens=toks)
    dt = time.perf_counter() - t0
    return len(toks) / dt, dt, len(toks)


# tokens per oracle call of the CPU baseline (the NVFP4 oracle quantises every
# expert matrix the sample touches, so its calls stay small)
CPU_SAMPLE_TOKENS = {"tiny_f32": 64, "std_moe_bf16": 128, "ultra_decode": 32, "ultra_zipf": 32,
                     "ultra_nvfp4": 4, "ultra_decode_nvfp4": 4, "ultra_nvfp4_fp8shared": 4}


def oracle_sample(wl, inp, n_tokens: int, min_seconds: float = 10.0, max_calls: int = 10000):
    """Bounded CPU baseline: oracle calls on fresh seeded token samples until
    at least `min_seconds` of oracle time (or `max_calls` calls).
    Returns (tokens/s, seconds, tokens, calls)."""
    total_t, total_tok, calls = 0.0, 0, 0
    while calls < max_calls and (calls == 0 or total_t < min_seconds):
        _, dt, n = oracle_tokens_per_s(wl, inp, n_tokens, seed=calls)
        total_t += dt
        total_tok += n
        calls += 1
    return total_tok / total_t, total_t, total_tok, calls


def run_reference(args, wl):
    """Reference arm: the oracle on the host cores. Each step is one oracle
    call on a fresh seeded sample of the workload's tokens, of the same size
    as the CPU baseline's calls (CPU_SAMPLE_TOKENS), so the two measure the
    same thing."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    inp = LI.make_inputs(wl)
    per_step = min(args.cpu_sample or CPU_SAMPLE_TOKENS.get(wl.name, 32), wl.T)
    for i in range(args.warmup):
        oracle_tokens_per_s(wl, inp, per_step, seed=1000 + i)
    total_t, total_tok = 0.0, 0
    for i in range(args.steps):
        _, dt, n = oracle_tokens_per_s(wl, inp, per_step, seed=i)
        total_t += dt
        total_tok += n
    v = total_tok / total_t
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * total_t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(wl),
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"{args.steps} call(s) on {per_step} random tokens of the {wl.name} batch "
                                   f"each ({total_tok} tokens), full weights, fp64 NumPy ({total_t:.1f} s)"},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def max_over_ranks(values, device):
    """Element-wise maximum of per-rank timings across the process group
    (every rank takes part; all ranks get the result)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def workload_config(wl):
    """The workload's description, identical in both arms."""
    c = {"workload": wl.name, "T": wl.T, "d": wl.d, "l": wl.l, "N": wl.N, "K": wl.K, "m": wl.m,
         "n_shared": wl.n_shared, "m_shared": wl.m_shared, "identity_projections": wl.identity,
         "zipf_bias": wl.zipf_bias, "outliers": wl.outliers, "parallelism": "replicas (one layer per GPU)",
         "l2": "no flush: weights alone exceed the 126 MB L2" if wl.dtype != "f32" else "tiny (fits L2)"}
    return c


# --------------------------------------------------------------------------
# our arm
# --------------------------------------------------------------------------
def run_backward(args, wl):
    """--backward: time lmoe_backward_nvfp4, the layer's backward pass with its
    routed experts under the NVFP4 training recipe (BF16 masters of every
    weight; one step = one backward over the workload's T tokens, inputs
    resident). Roofline: the six NVFP4 expert GEMMs (forward recompute, dgrad,
    wgrad of both layers) at the FP4 peak plus the BF16 GEMMs of the router,
    the projections and the shared experts at the BF16 peak, against the
    measured step. One JSON line, rank 0, N = 1."""
    import torch

    import latentmoe_fwd_b200 as L

    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
    inp = LI.make_inputs(wl)
    bits = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(
        torch.bfloat16).cuda()
    t = {k: bits(inp[k]) for k in ("x", "w_router", "w_down", "w_up", "w1", "w2", "ws1", "ws2")}
    bias = None if inp["router_bias"] is None else torch.from_numpy(inp["router_bias"]).cuda()
    cfg = L.config(T=wl.T, d=wl.d, l=wl.l, N=wl.N, K=wl.K, m=wl.m, n_shared=wl.n_shared, m_shared=wl.m_shared,
                   identity=wl.identity)
    w = L.weights(w_router=t["w_router"], router_bias=bias, w_down=t["w_down"], w_up=t["w_up"], w1=t["w1"],
                  w2=t["w2"], ws1=t["ws1"], ws2=t["ws2"])
    rng = np.random.default_rng(5)
    dout = bits(LI.bf16_bits(rng.standard_normal((wl.T, wl.d)) * 0.05))
    s_a = inp["a_global_scale"] if inp.get("a_global_scale") is not None else float(np.float32(256.0 / 2688.0))
    a_g = torch.tensor([s_a], dtype=torch.float32, device="cuda")
    bf = lambda *shape: torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    S, ms = wl.n_shared, wl.m_shared
    out = dict(dx=bf(wl.T, wl.d), dw_router=bf(wl.N, wl.d), dw1=bf(wl.N, wl.m, wl.l), dw2=bf(wl.N, wl.l, wl.m))
    if bias is not None:
        out["drouter_bias"] = torch.empty(wl.N, dtype=torch.float32, device="cuda")
    if not wl.identity:
        out.update(dw_down=bf(wl.l, wl.d), dw_up=bf(wl.d, wl.l))
    if S:
        out.update(dws1=bf(S, ms, wl.d), dws2=bf(S, wl.d, ms))
    g = L.grads(**out)
    ws = torch.zeros(int(L.lib.lmoe_backward_nvfp4_workspace(ctypes.byref(cfg))), dtype=torch.uint8, device="cuda")
    for _ in range(args.warmup):
        L.backward_nvfp4(cfg, w, t["x"], dout, a_g, 1, 0x5A5A, g, ws)
    torch.cuda.synchronize()
    stv, info = L.read_device_error(ws)
    if stv != L.OK:
        raise RuntimeError(f"device error during warm-up: {L.status_string(stv)} info={info:#x}")
    K = args.steps
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    stream = torch.cuda.current_stream()
    torch.cuda.synchronize()
    sampler = ClockSampler(torch.cuda.current_device())
    launches0 = L.kernel_launch_count()
    start.record(stream)
    for i in range(K):
        L.backward_nvfp4(cfg, w, t["x"], dout, a_g, 1 + i, 0x5A5A, g, ws, stream)
    end.record(stream)
    torch.cuda.synchronize()
    launches = L.kernel_launch_count() - launches0
    clocks = sampler.stop()
    stv, info = L.read_device_error(ws)
    if stv != L.OK:
        raise RuntimeError(f"device error in the timed region: {L.status_string(stv)} info={info:#x}")
    ms_step = start.elapsed_time(end) / K
    TK = wl.T * wl.K
    fp4_flops = 3 * 2 * (2.0 * TK * wl.l * wl.m)
    dense = 2.0 * wl.T * wl.d * wl.N * 3                      # router logits, dW_router, dx's router term
    if not wl.identity:
        dense += 2.0 * wl.T * wl.d * wl.l * 5                 # z, dc, dW_up, dW_down, dx's projection term
    if S:
        dense += 2.0 * wl.T * wl.d * S * ms * 5                # pre, dout Ws2, dWs2, dWs1, dx's shared term
    peaks, src = load_peaks()
    fp4_peak = 4.0 * peaks["bf16_tflops"]
    t_peak = fp4_flops / (fp4_peak * 1e9) + dense / (peaks["bf16_tflops"] * 1e9)
    line = {
        "metric": "LatentMoE layer backward tokens/s on 1 B200 (routed experts under the NVFP4 training recipe)",
        "value": wl.T / (ms_step * 1e-3), "unit": "tokens/s", "n_gpus": 1, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "dtype": "nvfp4+bf16", "data": "synthetic",
        "config": workload_config(wl),
        "roofline": {"bound": "tensor", "achieved_tflops": (fp4_flops + dense) / (ms_step * 1e9),
                     "fp4_flops": fp4_flops, "bf16_flops": dense, "time_at_peak_ms": t_peak,
                     "frac": t_peak / ms_step, "peak_fp4_tflops": fp4_peak, "peak_bf16_tflops": peaks["bf16_tflops"],
                     "peak_source": src,
                     "note": "grouped launches over all experts; the host reads their row counts once"},
        "gpu_launches": int(launches), "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(LI.WORKLOADS))
    ap.add_argument("--graph", action="store_true",
                    help="time replays of one forward captured in a CUDA graph (the e2e leg stays eager)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-sample", type=int, default=None, help="oracle tokens per call of cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override the workload's token count (smaller captures for ncu)")
    ap.add_argument("--experts", type=int, default=None,
                    help="override the workload's expert count (smaller captures for ncu)")
    ap.add_argument("--backward", action="store_true",
                    help="time the layer backward (NVFP4 training recipe for the routed experts) instead")
    args = ap.parse_args()
    wl = LI.WORKLOADS[args.workload]
    if args.tokens is not None:
        wl = LI.replace(wl, T=args.tokens)
    if args.experts is not None:
        wl = LI.replace(wl, N=args.experts)
    if args.impl == "reference":
        return run_reference(args, wl)
    if args.backward:
        return run_backward(args, wl)

    import torch
    import torch.distributed as dist

    import latentmoe_fwd_b200 as L

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    t_gen = time.perf_counter()
    inp = LI.make_inputs(wl)
    log(f"[bench] inputs for {wl.name} generated in {time.perf_counter() - t_gen:.1f}s")
    st = "f32" if wl.dtype == "f32" else "bf16"

    def dev(a):
        if a is None:
            return None
        if st == "f32":
            return torch.from_numpy(np.ascontiguousarray(a)).cuda()
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()

    t = {k: dev(inp[k]) for k in ("w_router", "w_down", "w_up", "w1", "w2", "ws1", "ws2")}
    bias = None if inp["router_bias"] is None else torch.from_numpy(inp["router_bias"]).cuda()
    tdtype = torch.float32 if st == "f32" else torch.bfloat16
    x_host = torch.from_numpy(np.ascontiguousarray(inp["x"]).view(np.int16 if st != "f32" else np.float32))
    x_host = (x_host.view(torch.bfloat16) if st != "f32" else x_host).pin_memory()
    x = x_host.cuda()
    out = torch.empty((wl.T, wl.d), dtype=tdtype, device="cuda")
    out_host = torch.empty((wl.T, wl.d), dtype=tdtype).pin_memory()
    cfg = L.config(T=wl.T, d=wl.d, l=wl.l, N=wl.N, K=wl.K, m=wl.m, n_shared=wl.n_shared, m_shared=wl.m_shared,
                   act=L.F32 if st == "f32" else L.BF16,
                   expert={"f32": L.F32, "bf16": L.BF16, "nvfp4": L.NVFP4}[wl.dtype], identity=wl.identity,
                   shared_fp8=wl.shared_fp8)
    extra = {}
    quant = None
    if wl.dtype == "nvfp4":
        # setup, not timed: NVFP4 expert weights (per-matrix global scale, MMA-tiled block scales)
        # the quantiser's own rate, on the BF16 W1 before it is replaced (outside the timed region)
        quant = quantizer_rates(L, t["w1"], load_peaks()[0]["hbm_gbs"]) if rank == 0 and world == 1 else None
        for key in ("w1", "w2"):
            codes, sf, gs = quantize_experts(L, t[key])
            t[key] = codes                         # the BF16 copy is released
            extra[key + "_sf"], extra[key + "_gs"] = sf, gs
        torch.cuda.empty_cache()
        extra["a_global_scale"] = torch.tensor([inp["a_global_scale"]], dtype=torch.float32, device="cuda")
        torch.cuda.synchronize()
    if wl.shared_fp8:
        # setup, not timed: FP8 shared-expert weights, one scale per stacked tensor
        S, ms, d = wl.n_shared, wl.m_shared, wl.d
        q = {}
        for key, rows, cols in (("ws1", S * ms, d), ("ws2", S * d, ms)):
            codes = torch.empty((rows, cols), dtype=torch.uint8, device="cuda")
            scale = torch.empty(1, dtype=torch.float32, device="cuda")
            qws = L.workspace(L.config(T=rows, d=cols, l=cols, N=1, K=1, m=cols), L.OP_FP8_QUANTIZE)
            L.fp8_quantize(t[key].reshape(rows, cols), L.BF16, rows, cols, None, codes, scale, qws)
            q[key], extra[key + "_scale"] = codes, scale
        t["ws1"], t["ws2"] = q["ws1"], q["ws2"]
        extra["shared_x_scale"] = torch.tensor([inp["shared_x_scale"]], dtype=torch.float32, device="cuda")
        extra["shared_h_scale"] = torch.tensor([inp["shared_h_scale"]], dtype=torch.float32, device="cuda")
        torch.cuda.synchronize()
    w = L.weights(w_router=t["w_router"], router_bias=bias, w_down=t["w_down"], w_up=t["w_up"], w1=t["w1"],
                  w2=t["w2"], ws1=t["ws1"], ws2=t["ws2"], **extra)
    ws = L.workspace(cfg, L.OP_FORWARD)
    stream = torch.cuda.current_stream()

    # routing statistics of this batch (outside any timed region)
    idx = torch.empty((wl.T, wl.K), dtype=torch.int32, device="cuda")
    gw = torch.empty((wl.T, wl.K), dtype=torch.float32, device="cuda")
    rws = L.workspace(cfg, L.OP_ROUTE)
    L.route(cfg, x, t["w_router"], bias, None, idx, gw, None, rws)
    counts = np.bincount(idx.cpu().numpy().reshape(-1), minlength=wl.N)
    alg_bytes, alg_flops, used, model_bytes = expert_gemm_work(wl, counts)

    for _ in range(args.warmup):
        L.forward(cfg, w, x, out, ws)
    stv, info = L.read_device_error(ws)
    if stv != L.OK:
        raise RuntimeError(f"device error during warm-up: {L.status_string(stv)} info={info:#x}")

    # --graph: one forward captured in a CUDA graph, replayed once per step
    graph, graph_launches = None, 0
    if args.graph:
        gs = torch.cuda.Stream()
        gs.wait_stream(stream)
        with torch.cuda.stream(gs):
            L.forward(cfg, w, x, out, ws, gs)   # first use on the capture stream
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        n0 = L.kernel_launch_count()
        with torch.cuda.graph(graph, stream=gs):
            L.forward(cfg, w, x, out, ws, gs)
        graph_launches = L.kernel_launch_count() - n0
        torch.cuda.synchronize()

    # ---- device-resident timed region ----
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(L.TRACE_EVENTS)] for _ in range(K)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(torch.cuda.current_device())
    time.sleep(0.05)
    launches0 = L.kernel_launch_count()
    start.record(stream)
    for i in range(K):
        if graph is not None:
            graph.replay()
        else:
            L.forward(cfg, w, x, out, ws, stream)
    end.record(stream)
    torch.cuda.synchronize()
    launches = L.kernel_launch_count() - launches0 + graph_launches * K
    clocks = sampler.stop()
    barrier()
    stv, info = L.read_device_error(ws)
    if stv != L.OK:
        raise RuntimeError(f"device error in the timed region: {L.status_string(stv)} info={info:#x}")
    ms = start.elapsed_time(end)
    # stage split: the same K forwards again, each recording timing events at
    # the library's stage boundaries on the launch stream (kept out of the
    # timed region: timing events serialise the kernel boundaries they mark)
    for i in range(K):
        L.forward_traced(cfg, w, x, out, ws, ev[i], stream)
    torch.cuda.synchronize()
    stv, info = L.read_device_error(ws)
    if stv != L.OK:
        raise RuntimeError(f"device error in the traced pass: {L.status_string(stv)} info={info:#x}")
    stage_ms = np.zeros(L.TRACE_EVENTS - 1)
    for i in range(K):
        for j in range(L.TRACE_EVENTS - 1):
            stage_ms[j] += ev[i][j].elapsed_time(ev[i][j + 1])
    stage_ms /= K

    # ---- end-to-end through host buffers ----
    # Every step copies its input from pinned host memory and its output back,
    # on copy streams of their own with two device buffers each way, so the
    # copies of step i overlap the forwards of steps i-1 and i+1 (the layout a
    # serving loop uses); the timed region spans the first copy in to the last
    # copy out.
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    x_buf = [x, torch.empty_like(x)]
    out_buf = [out, torch.empty_like(out)]
    out_hbuf = [out_host, torch.empty_like(out_host).pin_memory()]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_fwd = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    barrier()
    torch.cuda.synchronize()
    e_start.record(stream)
    h2d.wait_event(e_start)
    for i in range(K):
        b = i % 2
        if i >= 2:
            h2d.wait_event(ev_fwd[b])            # forward i-2 has read x_buf[b]
        with torch.cuda.stream(h2d):
            x_buf[b].copy_(x_host, non_blocking=True)
        ev_in[b].record(h2d)
        stream.wait_event(ev_in[b])
        if i >= 2:
            stream.wait_event(ev_out[b])         # out_buf[b] of step i-2 is on the host
        L.forward(cfg, w, x_buf[b], out_buf[b], ws, stream)
        ev_fwd[b].record(stream)
        d2h.wait_event(ev_fwd[b])
        with torch.cuda.stream(d2h):
            out_hbuf[b].copy_(out_buf[b], non_blocking=True)
        ev_out[b].record(d2h)
    for b in range(min(K, 2)):
        stream.wait_event(ev_out[b])
    e_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = e_start.elapsed_time(e_end)

    if world > 1:
        ms, e2e_ms = max_over_ranks([ms, e2e_ms], "cuda")

    tokens = wl.T * K * world
    value = tokens / (ms / 1000.0)
    e2e_value = tokens / (e2e_ms / 1000.0)

    peaks, peak_src = load_peaks()
    gemm_ms = stage_ms[3] + stage_ms[4]          # expert GEMM 1 + 2 (two launches)
    roof = roofline(wl, alg_bytes, alg_flops, gemm_ms, peaks, peak_src)
    roof.update({"kernel": expert_gemm_kernel(wl), "experts_used": used,
                 "traffic_model": model_bytes, "step_ms": ms / K})
    roof["traffic"] = traffic_record(wl.name)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n = args.cpu_sample or CPU_SAMPLE_TOKENS.get(wl.name, 32)
        v, dt, ntok, calls = oracle_sample(wl, inp, n)
        cpu = {"value": v, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"{calls} call(s) on {min(n, wl.T)} random tokens of the {wl.name} batch each "
                         f"({ntok} tokens), full weights, fp64 NumPy ({dt:.1f} s)"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms / K, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "fp32" if wl.dtype == "f32" else (
                ("nvfp4+fp8+bf16" if wl.shared_fp8 else "nvfp4+bf16") if wl.dtype == "nvfp4" else "bf16"),
            "data": "synthetic", "config": workload_config(wl),
            "roofline": roof, "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": int(x_host.numel() *
                                                                                     x_host.element_size()),
                    "d2h_bytes_per_step": int(out_host.numel() * out_host.element_size())},
            "gpu_launches": int(launches),
            "launch": "cuda_graph" if graph is not None else "stream",
            "clocks": clocks,
            "stage_ms": {n: float(v) for n, v in zip(L.TRACE_STAGES, stage_ms)},
        }
        if quant is not None:
            line["nvfp4_quantize"] = quant
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
