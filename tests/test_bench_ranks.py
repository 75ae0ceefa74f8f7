"""The multi-rank host logic of bench.py on CPU: two gloo ranks agree on the
slowest rank's times and on the whole-job throughput; the reference arm does
nothing on ranks other than 0."""
import importlib.util
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        b = _bench()
        ms = b.max_over_ranks({"step": 1.0 + rank, "fwd": 10.0 - rank, "bwd_main": 0.5 * (rank + 1)})
        out.put((rank, ms, b.job_tflops(world, 1e12, ms["step"])))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, value in got:
        assert ms == {"step": 2.0, "fwd": 10.0, "bwd_main": 1.0}
        assert value == pytest.approx(2 * 1e12 / 2e-3 / 1e12)  # 2 ranks x 1 TFLOP in 2 ms


def test_single_process_is_identity():
    b = _bench()
    assert b.max_over_ranks({"step": 3.5}) == {"step": 3.5}
    assert b.job_tflops(1, 2e12, 1.0) == pytest.approx(2000.0)


def test_reference_arm_is_silent_on_other_ranks(capsys):
    b = _bench()
    b.run_reference(None, 1, 2, b.WORKLOADS["b1_h32_s4096_d128_causal"])
    assert capsys.readouterr().out == ""
