"""Multi-process paths of bench.py on CPU (gloo; no GPU).

The decode is data parallel: with N GPUs every rank decodes its own replica
of the batch, and the job is timed by the slowest rank. These tests cover the
host-side pieces of that: the max-over-ranks reduction of timings and the
whole-job value, with two gloo ranks, and the reference arm launched by
torch.distributed.run with two ranks (rank 0 alone runs and prints).
"""

import importlib.util
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        bench = _bench()
        # rank r reports (r + 1) ms for the step and (10 - r) ms for the kernel
        got = bench.max_over_ranks([rank + 1.0, 10.0 - rank], world, torch.device("cpu"))
        q.put((rank, got, bench.job_value(world, 1000, got[0])))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, value in results:
        assert got == [2.0, 10.0], (rank, got)
        # 2 replicas x 1000 KV tokens in 2 ms (the slowest rank) = 1e6 tokens/s
        assert value == pytest.approx(1.0e6)


def test_single_process_reduction_is_identity():
    bench = _bench()
    assert bench.max_over_ranks([3.0, 4.5], 1, torch.device("cpu")) == [3.0, 4.5]
    assert bench.job_value(1, 500, 0.5) == pytest.approx(1.0e6)


def test_reference_arm_under_torchrun_two_ranks():
    """`bench.py --impl reference` as the driver launches it for N=2: one JSON
    line from rank 0, every rank exits 0."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3",
           "--workload", "C1"]
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [json.loads(l) for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, res.stdout
    line = lines[0]
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["value"] > 0 and line["e2e"]["value"] == line["value"]
    assert line["cpu_baseline"]["kind"] == "oracle"
    # the same config object the GPU arm prints for this workload (so the two
    # lines compare as one configuration)
    bench = _bench()
    sys.path.insert(0, ROOT)
    from mla_latent_kv_26_b200.workloads import make_inputs

    inp = make_inputs("C1")
    assert line["config"] == bench.decode_config(inp, bench.accounting(inp), 2, bench.l2_bytes_of())
    assert "l2" in line["config"] and line["config"]["parallelism"] == "replicas x2"


@pytest.mark.parametrize("op,extra", [("insert", ["--insert-batch", "2", "--insert-tokens", "64"]),
                                      ("absorb", ["--absorb-tokens", "2"])])
def test_widened_rows_reference_arm(op, extra):
    """`bench.py --op insert|absorb --impl reference`: one JSON line with the
    contract's keys, the oracle timed on the host (no GPU needed)."""
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--op", op, "--impl", "reference", "--steps", "1",
           "--warmup", "3"] + extra
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [json.loads(l) for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, res.stdout
    line = lines[0]
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["dtype"] == "f64"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0


def test_insert_and_absorb_accounting():
    """Algorithmic bytes of the widened rows, from their definitions: the
    insert moves each token's 1152-byte row in and out plus 8 index bytes,
    one cos/sin row per distinct position and one table entry per distinct
    (sequence, page); the projections read each weight half once."""
    bench = _bench()
    sys.path.insert(0, ROOT)
    from mla_latent_kv_26_b200.workloads import insert_inputs

    d = insert_inputs(lens=[130, 70], new_tokens=[130, 6], seed=1)
    acc = bench.insert_accounting(d)
    pages = 3 + 1  # positions 0..129 of sequence 0 span 3 pages, 64..69 of sequence 1 one page
    assert acc["tokens"] == 136
    assert acc["bytes"] == 136 * (2 * 1152 + 8) + 130 * 256 + pages * 4 + 1024
    a = bench.absorb_accounting(64, 128)
    assert a["absorb"] == 128 * 128 * 512 * 2 + 64 * 128 * (192 + 576) * 2
    assert a["unabsorb"] == 128 * 128 * 512 * 2 + 64 * 128 * (512 + 128) * 2
    assert a["flops"] == 2 * 2 * 64 * 128 * 128 * 512
