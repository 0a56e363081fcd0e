"""The multi-rank host logic of bench.py on two gloo ranks (CPU only).

Heads and batches of the layer are independent, so N GPUs run N copies of
the workload with no collective on the data path; the only cross-rank steps
are the barriers around the timed region and the max over ranks of the
elapsed time.  These run here with world_size 2 on the gloo backend.
"""
import os
import socket
import sys

import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import time

    import bench
    # rank 1 is slower: every rank must report rank 1's time
    ms = bench.timed_region(lambda i: time.sleep(0.02 * (1 + 4 * rank)), 3, world, "cpu")
    w, r, _ = bench._dist()
    out[rank] = (ms, w, r, bench._max_over_ranks(float(rank + 7), world, "cpu"))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_time_is_max_over_ranks():
    port = _free_port()
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.start_processes(_worker, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
    (ms0, w0, r0, m0), (ms1, w1, r1, m1) = out[0], out[1]
    assert (w0, r0, w1, r1) == (2, 0, 2, 1)
    assert ms0 == ms1  # both ranks hold the max
    assert ms0 >= 3 * 0.02 * 5 * 1e3 * 0.95  # rank 1 slept 0.1 s per step
    assert m0 == m1 == 8.0
