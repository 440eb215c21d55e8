"""The multi-GPU mode's host logic (replica ranks, slowest-rank timing, job throughput)
on two CPU processes with the gloo backend: no GPU, no layer data."""

import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

from linear_attention_layer_gated_b200 import replicas

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    r, w, lr = replicas.rank_info()
    replicas.init(w, lr, backend="gloo", timeout_s=60)
    try:
        local_ms = 1.0 + 2.5 * r             # rank 1 is the slower one
        slowest = replicas.max_over_ranks(local_ms, w)
        replicas.barrier(w)
        rate = replicas.job_throughput(8192, w, slowest * 1e-3)
        out.put((r, w, lr, slowest, rate))
    finally:
        replicas.finish(w)


def test_two_gloo_ranks_agree_on_the_slowest_time_and_the_job_rate():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=5) for _ in range(world))
    for r, (rank, w, lr, slowest, rate) in enumerate(res):
        assert (rank, w, lr) == (r, world, r)
        assert slowest == pytest.approx(3.5)                      # max over ranks, on every rank
        assert rate == pytest.approx(2 * 8192 / 3.5e-3)           # all ranks' tokens / slowest time


def test_single_process_defaults():
    assert replicas.rank_info({}) == (0, 1, 0)
    replicas.init(1, 0)  # no process group for one rank
    assert replicas.max_over_ranks(2.0, 1) == 2.0
    assert replicas.job_throughput(100, 1, 0.5) == 200


def test_reference_arm_other_ranks_do_no_work(capsys):
    sys.path.insert(0, ROOT)
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)

    class Args:
        steps, warmup = 1, 0
    assert bench.reference_arm(Args, rank=1, world=2) == 0  # only rank 0 runs and prints
    assert capsys.readouterr().out == ""
