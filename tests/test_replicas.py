"""The N > 1 path of bench.py on CPU: world-size-2 gloo ranks.

The forward has no exchange step, so N GPUs run N independent replicas; the
only collective is the max over ranks of the timed device milliseconds."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    import synth
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms, value = bench.aggregate(10.0 + 3.0 * rank, world, 64, 5)
        cfg = synth.CONFIGS[0]
        _, x = synth.make_inputs(cfg, 4, seed=bench.rank_seed(0, rank))
        q.put((rank, ms, value, x.tobytes()))
    finally:
        dist.destroy_process_group()


def test_two_replicas_max_over_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, ms0, v0, x0), (r1, ms1, v1, x1) = res
    # both ranks report the slowest rank's time and the whole job's tokens
    assert ms0 == ms1 == 13.0
    assert v0 == v1 == pytest.approx(2 * 64 * 5 / 0.013)
    # each replica processes its own batch
    assert x0 != x1


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    ms, value = bench.aggregate(8.0, 1, 16, 4)
    assert ms == 8.0 and value == pytest.approx(16 * 4 / 0.008)
    assert bench.rank_seed(3, 0) == 3 and bench.rank_seed(3, 2) == 2003
    assert np.isfinite(value)
