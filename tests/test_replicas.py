"""Multi-GPU layout is replicas only (independent sequences per GPU, no
collective on the decode path).  The host-side reduction of the benchmark's
statistics is checked here with two gloo ranks on the CPU."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    import sys
    import datetime
    import torch
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    tokens = [30, 50][rank]
    ms = [100.0, 125.0][rank]
    e2e = [200.0, 180.0][rank]
    out[rank] = bench.reduce_replicas(tokens, ms, e2e, world, torch.device("cpu"))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_reduction():
    mgr = mp.get_context("spawn").Manager()   # no fork of a multi-threaded parent
    out = mgr.dict()
    port = _free_port()
    mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
    for r in (0, 1):
        tokens, ms, e2e = out[r]
        assert tokens == 80            # tokens of all replicas
        assert ms == 125.0             # the slowest replica's time
        assert e2e == 380.0            # end-to-end throughputs add
    # the job's throughput: 80 tokens / 0.125 s
    assert 80 / 0.125 == 640.0


def test_single_rank_is_identity():
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    assert bench.reduce_replicas(7, 3.5, 9.0, 1, None) == (7, 3.5, 9.0)
