"""Host logic of the multi-replica bench (`bench.py --gpus N`): the path has
no exchange step, so N processes run independent replicas and the only
collective is the max over ranks of the device-timed step time.  Checked
here with two `gloo` ranks on the CPU."""
import importlib.util
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    sys.path.insert(0, ROOT)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, times, out):
    import datetime

    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        b = _bench()
        ms = b.reduce_max_over_ranks(times[rank], world, "cpu")
        out[rank] = (ms, b.whole_job_tokens_per_s(world, 8192, ms))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_value_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    port = _free_port()
    times = [1.25, 1.75]                      # rank 1 is the slower replica
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_rank, args=(r, 2, port, times, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        res = dict(out)
    for r in range(2):
        ms, value = res[r]
        assert ms == pytest.approx(1.75)
        # two replicas of 8192 tokens each per 1.75 ms step
        assert value == pytest.approx(2 * 8192 / 1.75e-3)


def test_single_rank_needs_no_collective():
    b = _bench()
    assert b.reduce_max_over_ranks(2.5, 1, "cpu") == 2.5
    assert b.whole_job_tokens_per_s(1, 8192, 2.0) == pytest.approx(8192 / 2e-3)


def test_kernel_hash_ignores_comments_only():
    import bench
    src = "int a; // note\n/* block\n comment */ int b;\n\n  // indented\nint c; /* tail */\n"
    assert bench.code_without_comments(src) == "int a;\n int b;\nint c;"
    reworded = src.replace("note", "other words").replace("block", "blk")
    assert bench.code_without_comments(reworded) == bench.code_without_comments(src)
    assert bench.code_without_comments(src.replace("int b", "int bb")) != \
        bench.code_without_comments(src)
