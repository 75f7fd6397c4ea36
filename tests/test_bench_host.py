"""Host-side logic of bench.py, on CPU: the max-over-ranks reduction under a
2-rank gloo process group, and the reference arm (the timed oracle) with its
rank behaviour under torchrun."""
import json
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    res = bench.max_over_ranks([1.0 + rank, 10.0 * (world - rank)], "cpu")
    out[rank] = res
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world = 2
    port = 29600 + os.getpid() % 300
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert out[0] == [2.0, 20.0] and out[1] == [2.0, 20.0]


def _run_bench(args, env_extra):
    env = dict(os.environ)
    env.update(env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, capture_output=True,
                          text=True, env=env, timeout=300, cwd=ROOT)


def test_reference_arm_prints_one_line_on_rank0():
    r = _run_bench(["--impl", "reference", "--workload", "tiny_f32", "--steps", "2", "--warmup", "1"],
                   {"RANK": "0", "WORLD_SIZE": "1"})
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["config"]["workload"] == "tiny_f32"


def test_reference_arm_other_ranks_exit_quietly():
    r = _run_bench(["--impl", "reference", "--workload", "tiny_f32", "--steps", "2", "--warmup", "1"],
                   {"RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_cpu_baseline_sample_is_time_bounded():
    sys.path.insert(0, ROOT)
    import bench
    import lmoe_inputs as LI
    wl = LI.WORKLOADS["tiny_f32"]
    inp = LI.make_inputs(wl)
    v, dt, ntok, calls = bench.oracle_sample(wl, inp, 16, min_seconds=0.2, max_calls=1000)
    assert calls >= 2 and ntok == 16 * calls       # repeated until the time bound
    assert dt >= 0.2 or calls == 1000
    assert v == pytest.approx(ntok / dt)
    _, _, ntok1, calls1 = bench.oracle_sample(wl, inp, 16, min_seconds=1e9, max_calls=3)
    assert calls1 == 3 and ntok1 == 48              # and by the call cap
    assert set(bench.CPU_SAMPLE_TOKENS) == set(LI.WORKLOADS)


def test_reference_arm_config_matches_our_arm():
    """Both arms describe the workload with the same dict (the driver compares them)."""
    sys.path.insert(0, ROOT)
    import bench
    import lmoe_inputs as LI
    for name in LI.WORKLOADS:
        c = bench.workload_config(LI.WORKLOADS[name])
        assert c["workload"] == name and "l2" in c


def test_expert_gemm_work_counts_weights_once_and_flops_by_definition():
    sys.path.insert(0, ROOT)
    import numpy as np
    import bench
    import lmoe_inputs as LI
    wl = LI.WORKLOADS["ultra_zipf"]
    counts = np.zeros(wl.N, dtype=np.int64)
    counts[:3] = [1000, 10, 1]                      # three experts used, 1011 rows
    b, f, used, model = bench.expert_gemm_work(wl, counts)
    assert used == 3
    assert b == 3 * 2 * wl.m * wl.l * 2             # W1_e and W2_e of the used experts, BF16
    assert f == 2.0 * 1011 * wl.l * wl.m * 2
    assert model == 1011 * (wl.l + wl.m) * 2 * 2    # z in, a out, a in, y out: not algorithmic
    wq = LI.WORKLOADS["ultra_nvfp4"]
    bq, _, _, _ = bench.expert_gemm_work(wq, counts)
    assert bq == 3 * 2 * wq.m * wq.l * (0.5 + 1 / 16)


def test_roofline_uses_burst_peaks_and_the_binding_roof():
    sys.path.insert(0, ROOT)
    import bench
    import lmoe_inputs as LI
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    wl = LI.WORKLOADS["ultra_zipf"]
    r = bench.roofline(wl, 4e9, 3.2e12, 2.0, peaks, "measured")
    assert r["bound"] == "tensor" and r["peak"] == 1600.0
    assert r["achieved"] == pytest.approx(3.2e12 / 2e-3 / 1e12)
    assert r["frac"] == pytest.approx(1600.0 / 1600.0)
    assert r["frac_of_sustained"] == pytest.approx(1600.0 / 1400.0)
    rq = bench.roofline(LI.WORKLOADS["ultra_nvfp4"], 1.2e9, 1.5e12, 0.5, peaks, "measured")
    assert rq["bound"] == "tensor" and rq["peak"] == 6400.0          # 4 x BF16 burst
    rd = bench.roofline(LI.WORKLOADS["ultra_decode"], 3e9, 6e9, 0.5, peaks, "fallback")
    assert rd["bound"] == "hbm" and rd["frac"] == pytest.approx(3e9 / 0.5e-3 / 1e9 / 6000.0)
