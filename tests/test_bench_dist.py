"""The N > 1 path of bench.py on CPU: two gloo ranks.

Each rank runs its own replica of the workload; the time that counts is the
max over ranks and `value` counts every rank's bytes.  This checks those
reductions with ranks that report different times, plus the reference arm's
rule that only rank 0 does work.
"""
import multiprocessing as mp
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms_local = 10.0 + 5.0 * rank
        ms = bench.reduce_max(ms_local, torch.device("cpu"))
        gbs = bench.whole_job_gbs(world, 1_000_000, 100, ms)
        q.put((rank, ms, gbs))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_value():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    results = sorted(q.get(timeout=5) for _ in range(world))
    for rank, ms, gbs in results:
        assert ms == 15.0                       # the slowest rank's time
        assert gbs == pytest.approx(2 * 1e6 * 100 / 15e-3 / 1e9)  # both ranks' bytes


def test_single_process_reduction_is_identity():
    import torch
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(3.5, torch.device("cpu")) == 3.5
    assert bench.whole_job_gbs(1, 2e9, 10, 1000.0) == pytest.approx(20.0)


def test_reference_arm_nonzero_ranks_exit_without_work():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True,
                       text=True, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_reference_arm_prints_contract_line():
    import json
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--steps", "2", "--warmup", "3"],
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "impl", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"


def test_algorithmic_bytes_hand_values():
    """The roofline numerator: input read once, output written once, filters
    and bias read once (hand arithmetic for the headline shapes)."""
    import bench
    from depthwise_convolution_fwd_b200.workloads import Case
    # MobileNet stride-2 layer: 32x56x56x144 -> 28x28, float32
    c = Case("m3", 32, 56, 56, 144, 3, 3, stride=2, padding=1)
    x, y = 32 * 56 * 56 * 144 * 4, 32 * 28 * 28 * 144 * 4
    assert bench.algorithmic_bytes(c, 28, 28, "fwd") == x + y + 144 * 9 * 4 + 144 * 4
    assert bench.algorithmic_bytes(c, 28, 28, "bwd") == x + y + 144 * 9 * 4
    assert bench.algorithmic_bytes(c, 28, 28, "wgrad") == x + y + 144 * 9 * 4 + 144 * 4
    assert bench.algorithmic_bytes(c, 28, 28, "fused") == x + y + 144 * 9 * 4 + 144 * 4 + 16 * 144
    # 512x512x256 3x3 with float16 weights and bfloat16 activations
    c = Case("l", 1, 512, 512, 256, 3, 3, wtype="f16")
    a = 512 * 512 * 256
    assert bench.algorithmic_bytes(c, 512, 512, "fwd", esz=2) == 2 * (2 * a) + 256 * 9 * 2 + 256 * 4
    # channel multiplier 2: 128 input channels, 256 outputs and filters
    c = Case("m", 1, 512, 512, 128, 3, 3, multiplier=2)
    assert bench.algorithmic_bytes(c, 512, 512, "bwd") == 4 * (512 * 512 * (128 + 256)) + 256 * 9 * 4
