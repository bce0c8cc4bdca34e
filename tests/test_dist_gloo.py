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
    mgr = mp.get_context("spawn").Manager()  # no fork of a threaded parent
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    t0, g0, idx0, _ = out[0]
    t1, g1, idx1, ref1 = out[1]
    assert t0 == t1 == 3.5                      # max over ranks
    assert g0 == g1 and g0[0] != g0[1]          # every rank sees both digests; batches differ
    assert idx0 == idx1 == [3, 77, 130, 201]    # same prepacked outlier set
    assert ref1 is None                         # only rank 0 runs the reference arm


def _tp_worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import mixed_precision_quantized_mixq_b200 as mq
        import synth
        from helpers import oracle_layer
        M, K, N, k_out = 8, 512, 512, 16
        idx = synth.outlier_channels(K, k_out)
        X = synth.activations(M, K, idx, synth.channel_factors(k_out))
        W = synth.weights(N, K)
        n0, n1 = mq.column_shard(N, rank, world)
        # this rank's output channels (the oracle stands in for the CUDA layer on CPU)
        y_local = oracle_layer(X, W[n0:n1], idx, "w8", synth.THRESHOLD)["y"].astype(np.float16)
        Y = mq.gather_columns(torch.from_numpy(y_local), world)
        out[rank] = Y.numpy().view(np.uint16).tobytes()
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks_column_split():
    # N-split (column-parallel) layer: each rank holds N/2 output channels, the
    # all-gather assembles the full output, identical to the unsplit layer
    import mixed_precision_quantized_mixq_b200 as mq
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import synth
    from helpers import oracle_layer
    world = 2
    mgr = mp.get_context("spawn").Manager()  # no fork of a threaded parent
    out = mgr.dict()
    mp.spawn(_tp_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    M, K, N, k_out = 8, 512, 512, 16
    idx = synth.outlier_channels(K, k_out)
    X = synth.activations(M, K, idx, synth.channel_factors(k_out))
    y = oracle_layer(X, synth.weights(N, K), idx, "w8", synth.THRESHOLD)["y"].astype(np.float16)
    assert out[0] == out[1] == y.view(np.uint16).tobytes()
    assert mq.column_shard(11008, 1, 2) == (5504, 11008)
    with pytest.raises(ValueError):
        mq.column_shard(4096, 0, 3)
