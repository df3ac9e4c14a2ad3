"""The multi-rank plumbing of bench.py on CPU: two gloo ranks (the benchmark runs
one replica per GPU and reports every rank's FLOPs over the slowest rank)."""
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


def _rank_main(rank, world, port, results):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    b = _bench()
    r, w, lr = b.dist_env()
    ms = 10.0 + 5.0 * rank                       # rank 1 is the slow one
    t_max = b.max_over_ranks(ms, w)
    results[rank] = (r, w, lr, t_max, b.whole_job_tflops(2.0e12, w, t_max))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    world = 2
    mgr = mp.Manager()
    results = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), results), nprocs=world,
                       start_method="spawn", join=True)
    for rank in range(world):
        r, w, lr, t_max, tflops = results[rank]
        assert (r, w, lr) == (rank, world, rank)
        assert t_max == 15.0
        assert tflops == pytest.approx(2.0e12 * 2 / 0.015 / 1e12)


def test_single_rank_is_identity():
    b = _bench()
    assert b.max_over_ranks(3.5, 1) == 3.5
    assert b.whole_job_tflops(1e12, 1, 1000.0) == pytest.approx(1.0)
