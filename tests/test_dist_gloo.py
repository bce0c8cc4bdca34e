"""The multi-rank host logic of bench.py on CPU: two gloo ranks.

Each rank processes its own seeded batch (weak scaling, no data-path
collective); timings are combined as the maximum over ranks; only rank 0
runs the CPU-oracle reference arm."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import synth
        (case,) = synth.tiny()
        X, idx = bench.rank_activations(case, rank)
        # per-rank "timings": the slowest rank decides
        t = bench.max_over_ranks(1.0 + 2.5 * rank, world)
        # distinct batches across ranks, same outlier channels
        digest = torch.tensor([float(np.abs(X.astype(np.float64)).sum())], dtype=torch.float64)
        gathered = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(gathered, digest)
        args = bench.main.__globals__["argparse"].Namespace(
            workload="tiny", case=None, modes=None, steps=1, warmup=1)
        ref = bench.run_reference(args, rank, world) if rank != 0 else "skipped"
        out[rank] = (t, [g.item() for g in gathered], list(map(int, idx)), ref)
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    t0, g0, idx0, _ = out[0]
    t1, g1, idx1, ref1 = out[1]
    assert t0 == t1 == 3.5                      # max over ranks
    assert g0 == g1 and g0[0] != g0[1]          # every rank sees both digests; batches differ
    assert idx0 == idx1 == [3, 77, 130, 201]    # same prepacked outlier set
    assert ref1 is None                         # only rank 0 runs the reference arm
