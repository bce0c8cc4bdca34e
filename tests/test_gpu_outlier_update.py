"""Outlier set kept across decode steps (next row f3), CUDA path vs the oracle.

A step that detects outlier channels outside the prepacked set (flags[1] > 0)
grows the set by them (host merge) and rebuilds only the outlier weight columns
(device gather); the next step then finds no detection outside the set and its
layer output matches the oracle's layer with the grown set.
"""
import numpy as np
import pytest

import oracle
import synth
from helpers import assert_y_close, oracle_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    return torch


@pytest.mark.parametrize("mode", ["w8", "w4"])
@pytest.mark.parametrize("N,K,k_old,k_new", [(512, 1024, 0, 5), (4096, 4096, 32, 64),
                                             (384, 2048, 7, 130)])
def test_extract_outlier_weights_matches_prepack(torch_cuda, mode, N, K, k_old, k_new):
    import mixed_precision_quantized_mixq_b200 as mq
    torch = torch_cuda
    W = synth.weights(N, K)
    idx_old = synth.outlier_channels(K, k_old)
    idx_new = synth.outlier_channels(K, k_new)
    Wd = torch.from_numpy(W).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    w = mq.prepack(Wd, torch.from_numpy(idx_old).cuda(), mq.MIXQ_W8 if mode == "w8" else mq.MIXQ_W4G128,
                   status=status)
    w2 = mq.update_outliers(w, Wd, torch.from_numpy(idx_new).cuda(), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    _, _, W_out = oracle.prepack_w8(W, idx_new)
    np.testing.assert_array_equal(w2.W_out.cpu().numpy().view(np.uint16), W_out.view(np.uint16))
    assert w2.Wq is w.Wq and w2.s_w is w.s_w  # the codes are kept as they are


def test_extract_rejects_unsorted_idx(torch_cuda):
    import mixed_precision_quantized_mixq_b200 as mq
    torch = torch_cuda
    Wd = torch.from_numpy(synth.weights(256, 512)).cuda()
    w = mq.prepack(Wd, torch.zeros(0, dtype=torch.int32, device="cuda"))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    mq.update_outliers(w, Wd, torch.tensor([9, 5], dtype=torch.int32, device="cuda"), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 1


@pytest.mark.parametrize("mode", ["w8", "w4"])
@pytest.mark.parametrize("M,K,N", [(16, 4096, 4096), (1, 4096, 11008), (64, 11008, 4096)])
def test_outlier_set_grows_then_detection_stops(torch_cuda, mode, M, K, N):
    import mixed_precision_quantized_mixq_b200 as mq
    torch = torch_cuda
    T = synth.THRESHOLD
    true_idx = synth.outlier_channels(K, 64)
    X = synth.activations(M, K, true_idx, synth.channel_factors(64))
    W = synth.weights(N, K)
    idx0 = true_idx[::2].copy()  # the prepacked set knows half of the outlier channels
    Xd, Wd = torch.from_numpy(X).cuda(), torch.from_numpy(W).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    md = mq.MIXQ_W8 if mode == "w8" else mq.MIXQ_W4G128
    w = mq.prepack(Wd, torch.from_numpy(idx0).cuda(), md, status=status)
    q = mq.quantize_act(Xd, w.idx, T, status=status)
    torch.cuda.synchronize()
    flags = q.flags.cpu().numpy()
    assert flags[1] > 0  # detections outside the set
    idx1 = mq.merge_outliers(q.bitmap, w.idx, K)
    # the grown set is the union of the old set and every detected channel
    o_bitmap = oracle.quantize_act(X, idx0, T)[3]
    det = np.flatnonzero(np.unpackbits(o_bitmap.view(np.uint8), bitorder="little")[:K])
    np.testing.assert_array_equal(idx1.cpu().numpy(), np.union1d(idx0, det))
    w1 = mq.update_outliers(w, Wd, idx1, status=status)
    Y, q1 = mq.linear(Xd, w1, T, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert int(q1.flags[1].item()) == 0  # nothing detected outside the grown set
    o = oracle_layer(X, W, idx1.cpu().numpy(), mode, T)
    np.testing.assert_array_equal(q1.Xq.cpu().numpy(), o["Xq"])
    np.testing.assert_array_equal(q1.X_out.cpu().numpy().view(np.uint16), o["X_out"].view(np.uint16))
    assert_y_close(Y.cpu().numpy(), o["y"], f"{mode} M{M} K{K} N{N} after the update")
