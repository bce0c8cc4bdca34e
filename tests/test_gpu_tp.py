"""N-split (column-parallel) layer on one GPU: every shard's CUDA layer, run in
turn on the same device, then concatenated in rank order.

Each output channel is quantized on its own (per-row weight scale, per-row
4-bit groups), so a shard's prepack equals those rows of the full prepack and
its output equals those columns of the full output.  For the 8-bit and the
progressive 4-bit formats the INT32 sums are exact whatever K split a shard's
launch plan picks, so the assembled output is bit-identical to the unsplit
CUDA layer.  For the fp16-group-scale format the fp32 sum over groups follows
the launch's K split, so it is checked against the oracle within the layer
tolerance.  The collective that would assemble the shards across GPUs is the
plain all-gather of `gather_columns` (tested on CPU ranks); this test covers
the per-rank CUDA layer.
"""
import numpy as np
import pytest

import oracle
import synth
from helpers import assert_y_close, oracle_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    import mixed_precision_quantized_mixq_b200 as mq
    return torch, mq


def _sharded(torch, mq, Xd, Wd, idxd, mode, world, T):
    """Quantize once, run every rank's shard, assemble [M, N]."""
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    q = mq.quantize_act(Xd, idxd, T, status=status)
    parts = []
    for r in range(world):
        w = mq.prepack_shard(Wd, idxd, mode, r, world, status=status)
        parts.append(mq.gemm(q, w, status=status))
    full = mq.prepack(Wd, idxd, mode, status=status)
    Y_full = mq.gemm(q, full, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return torch.cat(parts, dim=1).cpu().numpy(), Y_full.cpu().numpy()


@pytest.mark.parametrize("M,N,K,world", [(16, 4096, 4096, 2), (16, 4096, 4096, 4),
                                         (1, 11008, 4096, 2), (64, 4096, 11008, 4),
                                         (512, 11008, 4096, 2), (2048, 4096, 4096, 4)])
@pytest.mark.parametrize("mode", ["w8", "w4"])
def test_column_shards_assemble_the_unsplit_layer(env, M, N, K, world, mode):
    torch, mq = env
    k_out = 64
    idx = synth.outlier_channels(K, k_out)
    X = synth.activations(M, K, idx, synth.channel_factors(k_out))
    W = synth.weights(N, K)
    Xd, Wd, idxd = (torch.from_numpy(a).cuda() for a in (X, W, idx))
    fmt = mq.MIXQ_W8 if mode == "w8" else mq.MIXQ_W4G128
    Y_tp, Y_full = _sharded(torch, mq, Xd, Wd, idxd, fmt, world, synth.THRESHOLD)
    # bit-identical to the unsplit CUDA layer
    np.testing.assert_array_equal(Y_tp.view(np.uint16), Y_full.view(np.uint16))
    # and within tolerance of the oracle on a window of tokens
    rows = (0, M) if M <= 16 else (M // 2 - 4, M // 2 + 4)
    y = oracle_layer(X, W, idx, mode, synth.THRESHOLD, rows)["y"]
    assert_y_close(Y_tp[rows[0]:rows[1]], y, f"{mode} M{M} N{N} K{K} P{world}")


@pytest.mark.parametrize("M,N,K,world", [(16, 4096, 4096, 4), (64, 11008, 4096, 2)])
def test_column_shards_fp16_group_scale(env, M, N, K, world):
    torch, mq = env
    k_out = 64
    idx = synth.outlier_channels(K, k_out)
    X = synth.activations(M, K, idx, synth.channel_factors(k_out))
    W = synth.weights(N, K)
    Xd, Wd, idxd = (torch.from_numpy(a).cuda() for a in (X, W, idx))
    Y_tp, Y_full = _sharded(torch, mq, Xd, Wd, idxd, mq.MIXQ_W4G128_F16S, world, synth.THRESHOLD)
    Xq, s_x, X_out, _, _ = oracle.quantize_act(X, idx, synth.THRESHOLD)
    _, _, W_out = oracle.prepack_w8(W, idx)
    q, s, z = oracle.prepack_w4b(W)
    y = oracle.linear_w4b(Xq, s_x, X_out, q, s, z, W_out)[1]
    assert_y_close(Y_tp, y, f"w4b M{M} N{N} K{K} P{world}")
    assert_y_close(Y_full, y, f"w4b unsplit M{M} N{N} K{K}")
