"""Multi-rank host logic of bench.py, on the CPU with the gloo backend (world size 2).

The attention path has no exchange between ranks: a multi-GPU run gives every
rank its own batch (weak scaling), and the only collectives are the barriers and
the max over ranks of the device timings. These tests cover that plumbing without
a GPU: the max-over-ranks reduction, the whole-job throughput formula, per-rank
seeding, and the reference arm under torchrun (rank 0 prints the one line).
"""
import datetime
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import fa_synth  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _max_worker(rank, world, port, queue):
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench as b

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # Rank r reports times (1 + r, 10 - r, r): the slowest rank differs per entry.
        out = b.max_over_ranks([1.0 + rank, 10.0 - rank, float(rank)], None, world)
        queue.put((rank, out))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_max_worker, args=(r, 2, port, queue)) for r in range(2)]
    for p in procs:
        p.start()
    results = dict(queue.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert results[0] == results[1] == [2.0, 10.0, 1.0]


def test_max_over_ranks_single_rank_is_identity():
    assert bench.max_over_ranks([3, 1.5], None, 1) == [3.0, 1.5]


def test_whole_job_throughput_is_weak_scaling():
    # 2 ranks, each 1e12 flop per step, 10 steps, slowest rank 1000 ms -> 20 TFLOP/s.
    assert bench.whole_job_tflops(1e12, 10, 2, 1000.0) == pytest.approx(20.0)
    # The same per-rank work on 8 ranks in the same time is 4x the 2-rank total.
    assert bench.whole_job_tflops(1e12, 10, 8, 1000.0) == pytest.approx(80.0)


def test_rank_batches_are_independent_and_reproducible():
    a0 = fa_synth.attention_input_bits(1, 2, 256, 64, "bf16", seed=bench.rank_seed(0))
    a1 = fa_synth.attention_input_bits(1, 2, 256, 64, "bf16", seed=bench.rank_seed(1))
    b0 = fa_synth.attention_input_bits(1, 2, 256, 64, "bf16", seed=bench.rank_seed(0))
    for name in ("q", "k", "v", "do"):
        assert np.array_equal(a0[name], b0[name])
        assert not np.array_equal(a0[name], a1[name])


def test_reference_arm_under_torchrun_prints_one_line_from_rank0():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0",
           "--workload", "gpt2_small", "--reference-seconds", "2"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference"
    assert line["n_gpus"] == 2
    assert line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle"


def test_gpus_flag_starts_its_own_ranks():
    # Without torchrun, --gpus 2 re-launches the script as two ranks itself: the
    # one printed line comes from rank 0 of a world of 2.
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "1",
           "--warmup", "0", "--workload", "gpt2_small", "--reference-seconds", "2"]
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    env["OMP_NUM_THREADS"] = "1"
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    assert json.loads(lines[0])["n_gpus"] == 2


def test_world_size_mismatch_fails_loudly():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0", OMP_NUM_THREADS="1")
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "1",
           "--warmup", "0", "--workload", "tiny_exact", "--reference-seconds", "1"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT, env=env)
    assert r.returncode != 0
    assert "WORLD_SIZE" in r.stderr
