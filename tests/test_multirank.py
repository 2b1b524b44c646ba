"""The N > 1 plumbing of bench.py on CPU: two gloo ranks on 127.0.0.1.
Barrier, max over ranks, the weak-scaling aggregate, and a rank that leaves
early: the other one must end with an error (a short process-group timeout),
not hang."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env(rank, world, port):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)


def _worker_ok(rank, world, port, out):
    _env(rank, world, port)
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_setup(world, backend="gloo", timeout_s=30)
    assert (w, r) == (world, rank)
    bench.barrier(w)
    out[rank] = bench.max_over_ranks(1.5 * (rank + 1), w)
    dist.destroy_process_group()


def _worker_leaves(rank, world, port, out):
    _env(rank, world, port)
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_setup(world, backend="gloo", timeout_s=5)
    bench.barrier(w)
    if rank == 1:
        out[rank] = "left"
        return                                   # between steps, nothing in flight
    try:
        bench.max_over_ranks(1.0, w)             # the peer is gone
        out[rank] = "no error"
    except Exception as e:                       # gloo timeout / connection closed
        out[rank] = "error: " + type(e).__name__
    finally:
        try:
            dist.destroy_process_group()
        except Exception:
            pass


def test_two_ranks_barrier_and_max():
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker_ok, args=(2, _free_port(), out), nprocs=2, start_method="spawn")
        assert out[0] == out[1] == 3.0


def test_rank_leaving_early_is_an_error_not_a_hang():
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker_leaves, args=(2, _free_port(), out), nprocs=2,
                           start_method="spawn")
        assert out[1] == "left"
        assert out[0].startswith("error"), out[0]


def test_weak_scaling_aggregate():
    sys.path.insert(0, ROOT)
    import bench
    # every rank runs the whole workload: throughput scales with the ranks
    # 1e13 ops in 10 ms on each rank = 1000 TOPS per rank
    assert bench.aggregate(1e13, 10.0, 1) == pytest.approx(1000.0)
    assert bench.aggregate(1e13, 10.0, 8) == pytest.approx(8000.0)
