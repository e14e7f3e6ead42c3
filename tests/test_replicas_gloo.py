"""The replica (N > 1) aggregation on CPU: two gloo ranks, max-over-ranks time,
whole-job throughput; and the benchmark's reference arm (the CPU oracle)."""
import json
import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank(rank, world, port, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from token_mixing_feature_b200 import replicas
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        local_ms = 100.0 + 50.0 * rank            # rank 1 is the slow one
        r = replicas.job_throughput(512, 10, local_ms, world)
        q.put((rank, r))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    out = dict(q.get(timeout=120) for _ in ps)
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in (0, 1):
        assert out[r]["elapsed_ms"] == 150.0
        assert out[r]["samples"] == 512 * 10 * 2
        assert abs(out[r]["samples_per_s"] - 10240 / 0.15) < 1e-6


def test_single_process_is_identity():
    sys.path.insert(0, ROOT)
    from token_mixing_feature_b200 import replicas
    r = replicas.job_throughput(64, 4, 8.0, 1)
    assert r["elapsed_ms"] == 8.0 and r["samples_per_s"] == 64 * 4 / 0.008


def test_bench_reference_arm_runs_on_cpu():
    env = dict(os.environ, OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny_f32", "--steps", "2", "--warmup", "3"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "samples/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
