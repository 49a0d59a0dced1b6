"""The N > 1 path of bench.py on CPU: world-size-2 gloo process group, the
replicas' timings aggregated as the max over ranks, throughput summed over ranks."""
import importlib.util
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench = _bench()
        # rank r measured (0.2 + 0.1 r) ms per step and (0.3 + 0.2 r) ms end to end
        res = bench.aggregate_over_ranks(0.2 + 0.1 * rank, 0.3 + 0.2 * rank, world, 32, "cpu")
        out[rank] = torch.tensor(res, dtype=torch.float64)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_step_and_sum_tokens():
    world = 2
    out = torch.zeros(world, 4, dtype=torch.float64).share_memory_()
    mp.start_processes(_rank, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    for r in range(world):
        ms, e2e, value, e2e_value = out[r].tolist()
        assert ms == pytest.approx(0.3) and e2e == pytest.approx(0.5)
        assert value == pytest.approx(2 * 32 / 0.3e-3)
        assert e2e_value == pytest.approx(2 * 32 / 0.5e-3)


def test_one_rank_is_its_own_max():
    bench = _bench()
    ms, e2e, value, e2e_value = bench.aggregate_over_ranks(0.25, 0.4, 1, 32, "cpu")
    assert (ms, e2e) == (0.25, 0.4) and value == pytest.approx(32 / 0.25e-3)
