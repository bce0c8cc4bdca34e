"""4-bit weights with an fp16 group scale and an integer zero (MixLLM reading),
CUDA path vs the oracle, through the C ABI (needs a B200).

Bit for bit: the codes q, the (s, z) pairs and W_out of the prepack, and the
INT32 sums of Xq * (q - z) (run through the progressive format's raw kernel
with every group scale set to 1, which expands each code to q - z).  Within
|Y - y| <= max(1e-3, 1e-2 |y|) of the oracle's fp64 value: the layer output,
whose per-group fp32 scaling and accumulation order the pages leave open.
"""
import numpy as np
import pytest

import oracle
import synth
from helpers import Gpu, assert_y_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gpu():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    return Gpu()


def _prepack(gpu, W, idx):
    torch, mq = gpu.torch, gpu.mq
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    w = mq.prepack(gpu.dev(W), gpu.dev(np.asarray(idx, np.int32)), mq.MIXQ_W4G128_F16S,
                   status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return w


def _pairs(w):
    """(s fp16 [N, K/128], z uint8 [N, K/128]) from the device group pairs [K/128, N, 2]."""
    g = w.grp.cpu().numpy()
    return np.ascontiguousarray(g[:, :, 0].T), np.ascontiguousarray(g[:, :, 1].T).astype(np.uint8)


@pytest.mark.parametrize("N,K,k_out", [(128, 128, 0), (256, 512, 4), (384, 1024, 130),
                                       (4096, 4096, 64)])
def test_prepack_matches_oracle(gpu, N, K, k_out):
    W = synth.weights(N, K)
    W[0, :128] = 0            # an all-zero group
    if K > 128:
        W[1, 128:256] = np.abs(W[1, 128:256]) + np.float16(0.01)  # an all-positive group
    W[2, :128] = np.float16(6e-8) * (np.arange(128) % 2)  # a range below the fp16 scale range
    idx = synth.outlier_channels(K, k_out)
    w = _prepack(gpu, W, idx)
    q_o, s_o, z_o = oracle.prepack_w4b(W)
    q, _, z2 = gpu.unpack_w4(w)
    s, z = _pairs(w)
    np.testing.assert_array_equal(q, q_o)
    np.testing.assert_array_equal(s.view(np.uint16), s_o.view(np.uint16))
    np.testing.assert_array_equal(z, z_o)
    np.testing.assert_array_equal(z2, z_o)
    if k_out:
        _, _, W_out = oracle.prepack_w8(W, idx)
        np.testing.assert_array_equal(w.W_out.cpu().numpy().view(np.uint16), W_out.view(np.uint16))
    assert w.s_w is None


@pytest.mark.parametrize("M,N,K", [(1, 256, 512), (16, 4096, 4096), (130, 384, 1024)])
def test_int32_sums_of_q_minus_z(gpu, M, N, K):
    """sum_k Xq (q - z) over all K equals the sum of the oracle's per-group partials."""
    torch, mq = gpu.torch, gpu.mq
    W = synth.weights(N, K)
    w = _prepack(gpu, W, [])
    q_o, s_o, z_o = oracle.prepack_w4b(W)
    unit = w.grp.clone()
    unit[:, :, 0] = 1.0  # group scale 1: the progressive expansion gives q - z
    Xq = np.random.default_rng(M + N).integers(-127, 128, size=(M, K)).astype(np.int8)
    acc = torch.full((M, N), -7, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    mq.mixq_debug_gemm_i32(mq.MIXQ_W4G128, gpu.dev(Xq), w.Wq, unit, acc, N, 0, 0, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    part, _ = oracle.linear_w4b(Xq, np.ones(M, np.float32), None, q_o, s_o, z_o, None)
    np.testing.assert_array_equal(acc.cpu().numpy(), part.sum(axis=2))


def _layer(gpu, X, W, idx, T, flags_null=False):
    torch, mq = gpu.torch, gpu.mq
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    w = _prepack(gpu, W, idx)
    q = mq.quantize_act(gpu.dev(X), w.idx, T, status=status)
    M, K = X.shape
    Y = torch.full((M, w.N), float("nan"), dtype=torch.float16, device="cuda")
    mq.mixq_gemm_w4a8o16_f16s(M, w.N, K, w.k_out, q.Xq, q.s_x, q.X_out, w.Wq, w.grp, w.W_out,
                              None if flags_null else q.flags, Y, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return Y.cpu().numpy()


def _oracle_layer(X, W, idx, T, rows=None):
    Xq, s_x, X_out, _, _ = oracle.quantize_act(X, idx, T)
    _, _, W_out = oracle.prepack_w8(W, idx)
    q, s, z = oracle.prepack_w4b(W)
    xo = X_out if X_out.shape[1] else None
    wo = W_out if W_out.shape[1] else None
    m0, m1 = (0, X.shape[0]) if rows is None else rows
    return oracle.linear_w4b(Xq, s_x, xo, q, s, z, wo, m0, m1)[1]


@pytest.mark.parametrize("M,K,N,k_out", [(1, 2048, 512, 64), (16, 4096, 1024, 64),
                                         (24, 1024, 512, 16), (40, 2048, 384, 32),
                                         (64, 1024, 640, 64), (100, 512, 256, 4),
                                         (130, 768, 512, 130), (300, 1024, 256, 0),
                                         (16, 1024, 4096, 32), (8, 1024, 28672, 64),
                                         (16, 4096, 256, 0)])
def test_layer_within_tolerance(gpu, M, K, N, k_out):
    idx = synth.outlier_channels(K, k_out)
    X = synth.activations(M, K, idx, synth.channel_factors(k_out)) if k_out else \
        synth.activations(M, K)
    W = synth.weights(N, K)
    assert_y_close(_layer(gpu, X, W, idx, synth.THRESHOLD), _oracle_layer(X, W, idx, synth.THRESHOLD),
                   f"M{M} K{K} N{N} ko{k_out}")


@pytest.mark.parametrize("M", [48, 8])
def test_no_token_mixed_and_null_flags(gpu, M):
    K, N = 2048, 512
    idx = synth.outlier_channels(K, 64)
    X = synth.activations(M, K)  # unscaled: no token above T
    W = synth.weights(N, K)
    y = _oracle_layer(X, W, idx, synth.THRESHOLD)
    assert_y_close(_layer(gpu, X, W, idx, synth.THRESHOLD), y, "fast path")
    assert_y_close(_layer(gpu, X, W, idx, synth.THRESHOLD, flags_null=True), y, "flags NULL")


@pytest.mark.parametrize("M,N,K", [(16, 11008, 4096), (16, 4096, 11008), (2048, 4096, 4096)])
def test_full_size_sampled_rows(gpu, M, N, K):
    """Llama-shaped launches; the oracle computes a window of rows."""
    k_out = 64
    idx = synth.outlier_channels(K, k_out)
    X = synth.activations(M, K, idx, synth.channel_factors(k_out))
    W = synth.weights(N, K)
    Y = _layer(gpu, X, W, idx, synth.THRESHOLD)
    rows = (0, M) if M <= 16 else (M // 2 - 3, M // 2 + 3)
    assert_y_close(Y[rows[0]:rows[1]], _oracle_layer(X, W, idx, synth.THRESHOLD, rows),
                   f"M{M} N{N} K{K} rows {rows}")
