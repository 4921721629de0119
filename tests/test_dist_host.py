"""Host logic of the multi-rank benchmark (bench.py --gpus N under torchrun), run as two
gloo ranks on CPU: process-group setup, the max-over-ranks device time, the whole-job
throughput and the per-rank data shard. The data path itself has no collective: each
rank decodes its own sequences.
"""
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TESTS = os.path.dirname(os.path.abspath(__file__))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    from long_context_decode_lr_b200 import synth

    w_, r_, _ = bench.dist_setup(world, backend="gloo")
    ms = 2.0 + 3.0 * r_  # rank 1 is the slower one
    ms_max = bench.max_over_ranks(ms, w_)
    bench.barrier(w_)
    w = synth.WORKLOADS["tiny_1k"]
    wr = w.replace(seed=w.seed + bench.rank_seed_offset(r_))
    q = synth.queries(wr, synth.model_weights(wr), 0)
    value = bench.job_tokens_per_s(w.batch * w.T, w_, ms_max)
    out.put((r_, w_, ms_max, value, float(abs(q).sum())))
    dist.destroy_process_group()


def test_two_gloo_ranks_share_max_time_and_own_shards():
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    env_path = os.environ.get("PYTHONPATH", "")
    os.environ["PYTHONPATH"] = os.pathsep.join([ROOT, TESTS] + ([env_path] if env_path else []))
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    try:
        for p in procs:
            p.start()
        res = sorted(out.get(timeout=180) for _ in range(2))
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
        os.environ["PYTHONPATH"] = env_path
    assert [p.exitcode for p in procs] == [0, 0]
    (r0, w0, m0, v0, q0), (r1, w1, m1, v1, q1) = res
    assert (r0, r1, w0, w1) == (0, 1, 2, 2)
    assert m0 == m1 == 5.0                       # the slowest rank's time, on every rank
    assert v0 == v1 == pytest.approx(2 * 1024 / 5e-3)  # all ranks' tokens over that time
    assert q0 != q1                              # each rank decodes different sequences


def test_reference_arm_runs_on_rank_zero_only():
    sys.path.insert(0, ROOT)
    import bench

    class Args:
        workload, warmup, steps = "tiny_1k", 3, 1

    assert bench.run_reference(Args, world=2, rank=1) is None
