"""The N>1 bench path on the CPU: world-size-2 gloo ranks.

Decode sequences are independent, so `bench.py --gpus N` runs one set of layer replicas
per rank with no data-path collective (weak scaling).  What ranks exchange is timing:
the job's time is the slowest rank's, and the value counts every rank's units.  The
reference arm runs on rank 0 alone; other ranks exit without work.
"""

import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, local_ms, units, out_dir):
    import datetime

    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        T = bench.max_over_ranks(local_ms[rank], world, dist, "cpu")
        v = bench.job_value(units, world, T)
        dist.barrier()
        with open(os.path.join(out_dir, f"r{rank}.txt"), "w") as f:
            f.write(f"{T} {v}")
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_world1_is_identity():
    assert bench.max_over_ranks(3.25, 1) == 3.25


def test_job_value_weak_scaling():
    # 2 layers x 100 steps per rank, 4 ranks, slowest rank 50 ms -> 800 units / 0.05 s
    assert bench.job_value(200, 4, 50.0) == pytest.approx(16000.0)
    # doubling ranks at fixed per-rank work and time doubles the value
    assert bench.job_value(200, 8, 50.0) == pytest.approx(2 * bench.job_value(200, 4, 50.0))


def test_two_gloo_ranks_agree_on_slowest_time(tmp_path):
    world, units = 2, 1600
    local_ms = [11.0, 17.5]
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, local_ms, units, str(tmp_path)))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = [tuple(map(float, open(tmp_path / f"r{r}.txt").read().split())) for r in range(world)]
    for T, v in res:
        assert T == max(local_ms)
        assert v == pytest.approx(units * world / (max(local_ms) / 1e3))


def test_reference_arm_nonzero_rank_exits_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_prefill_work_matches_the_workload_arithmetic():
    # the 8,192-query chunk after 65,536 tokens: 142.6 M (query, entry) pairs for the indexer
    # (1.168 TFLOP in FP8 at 32 heads x 128 dims), 1,152 rows per query for the attention
    # (1.237 TFLOP in BF16 at 64 heads x 512 dims) and 9.66 GB of gathered bf16 rows
    from csa_synth import get_workload
    wl = get_workload("csa_prefill_8k")
    layer = wl.layers[0]
    prefix = wl.n - wl.Tq
    t = prefix + np.arange(wl.Tq)
    idx, att, gather = bench.prefill_work(layer, t, wl.n // layer.m, wl.B)
    pairs = sum(min((int(x) + 1) // layer.m, wl.n // layer.m) for x in t)
    assert abs(pairs - 142.6e6) < 0.05e6
    assert abs(idx - 1.168e12) < 0.001e12
    assert abs(att - 1.237e12) < 0.001e12
    assert abs(gather - 9.66e9) < 0.01e9


def test_kernel_hash_ignores_comments_but_not_code(tmp_path, monkeypatch):
    # the recorded DRAM traffic stays valid across comment edits of the indexer sources, and is
    # dropped (traffic null) once their code changes
    src = "__global__ void k(int* p) {  // writes one\n  /* block\n comment */ p[0] = 1;\n}\n"
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    f = tmp_path / "k.cu"
    f.write_text(src)
    h0 = bench.sha_of(["k.cu"])
    f.write_text(src.replace("writes one", "stores a 1").replace("block\n comment", "other words"))
    assert bench.sha_of(["k.cu"]) == h0
    f.write_text(src.replace("p[0] = 1", "p[0] = 2"))
    assert bench.sha_of(["k.cu"]) != h0
