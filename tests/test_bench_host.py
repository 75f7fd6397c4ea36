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
