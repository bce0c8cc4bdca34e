"""The persistent CTA-pair kernels (tcgen05 cta_group::2, two SMs per tile):
W8A8 with 256-token x 256-channel tiles and W4A8 (progressive 4-bit weights
expanded into tensor memory) with 256-channel x 256-token tiles, CUDA path vs
the oracle through the C ABI.

Raw INT32 accumulators bit for bit (exact integer sums) at shapes that cover
one tile, several tiles per pair, ragged token counts, and an odd number of
128-channel weight tiles (the last pair tile's second half out of range).
The layer (through the launch plan, which picks this kernel at large M)
within |Y - y| <= max(1e-3, 1e-2 |y|) of the oracle: with outliers (the
epilogue scales the INT32 product in tensor memory and the FP16 outlier
product is accumulated onto it), with no token mixed, and with flags NULL.
"""
import numpy as np
import pytest

import oracle
import synth
from helpers import Gpu, assert_y_close, oracle_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gpu():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    return Gpu()


def _codes(M, N, K, seed):
    rng = np.random.default_rng(seed)
    Xq = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    Wq = rng.integers(-127, 128, size=(N, K)).astype(np.int8)
    return Xq, Wq


@pytest.mark.parametrize("M,N,K", [(256, 256, 128), (512, 512, 1024), (300, 384, 512),
                                   (1000, 1280, 2048), (2048, 4096, 1024), (257, 4992, 256),
                                   (512, 256, 384)])
def test_pair_int32_bit_exact(gpu, M, N, K):
    torch, mq = gpu.torch, gpu.mq
    # weights through the real prepack (codes of W ~ N(0, 0.02)), tokens random codes
    W = synth.weights(N, K, seed=M + N)
    w = mq.prepack(gpu.dev(W), gpu.dev(np.zeros(0, np.int32)), mq.MIXQ_W8)
    Wq8 = gpu.unpack_w8(w)
    Xq = np.random.default_rng(M * 7 + K).integers(-127, 128, size=(M, K)).astype(np.int8)
    acc = gpu.acc_i32(Xq, w, bn=512)
    rows = (0, M) if M * N * K <= 2 ** 31 else (M // 2 - 8, M // 2 + 8)
    want = oracle.gemm_i32(Xq, Wq8, *rows)
    np.testing.assert_array_equal(acc[rows[0]:rows[1]], want)
    if rows != (0, M):
        # last rows too (the ragged tail of the last token tile)
        np.testing.assert_array_equal(acc[M - 8:], oracle.gemm_i32(Xq, Wq8, M - 8, M))


def test_pair_int32_matches_the_128_tile_kernel(gpu):
    M, N, K = 1536, 11008, 4096
    W = synth.weights(N, K)
    torch, mq = gpu.torch, gpu.mq
    w = mq.prepack(gpu.dev(W), gpu.dev(np.zeros(0, np.int32)), mq.MIXQ_W8)
    Xq = gpu.dev(np.random.default_rng(3).integers(-127, 128, size=(M, K)).astype(np.int8))
    np.testing.assert_array_equal(gpu.acc_i32(Xq, w, bn=512), gpu.acc_i32(Xq, w, bn=128))


def _plan_is_pair(mq, M, N, K):
    bn, split, ctas = mq.mixq_gemm_plan(mq.MIXQ_W8, M, N, K)
    return bn == 256


@pytest.mark.parametrize("M,N,K,k_out", [(1024, 5120, 1024, 64), (1280, 4992, 2048, 256),
                                         (1024, 5120, 1024, 0), (2048, 11008, 4096, 128),
                                         (300, 640, 384, 32), (512, 28672, 8192, 128)])
def test_pair_layer_within_tolerance(gpu, M, N, K, k_out):
    mq = gpu.mq
    assert _plan_is_pair(mq, M, N, K)
    idx = synth.outlier_channels(K, k_out)
    X = synth.activations(M, K, idx, synth.channel_factors(k_out)) if k_out else \
        synth.activations(M, K)
    W = synth.weights(N, K)
    g = gpu.layer(X, W, idx, "w8", synth.THRESHOLD)
    assert g["status"] == 0
    rows = (0, M) if M * N * K <= 2 ** 33 else (M // 2 - 6, M // 2 + 6)
    o = oracle_layer(X, W, idx, "w8", synth.THRESHOLD, rows)
    assert_y_close(g["Y"][rows[0]:rows[1]], o["y"], f"pair M{M} N{N} K{K} ko{k_out}")
    if rows != (0, M):
        o2 = oracle_layer(X, W, idx, "w8", synth.THRESHOLD, (M - 4, M))
        assert_y_close(g["Y"][M - 4:], o2["y"], "last rows")


def test_pair_layer_no_token_mixed_and_null_flags(gpu):
    torch, mq = gpu.torch, gpu.mq
    M, N, K, k_out = 1024, 5120, 1024, 64
    idx = synth.outlier_channels(K, k_out)
    W = synth.weights(N, K)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    w = mq.prepack(gpu.dev(W), gpu.dev(idx), mq.MIXQ_W8, status=status)
    for X, flags_null in ((synth.activations(M, K), False),
                          (synth.activations(M, K, idx, synth.channel_factors(k_out)), True)):
        q = mq.quantize_act(gpu.dev(X), w.idx, synth.THRESHOLD, status=status)
        Y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        mq.mixq_gemm_w8a8o16(M, N, K, k_out, q.Xq, q.s_x, q.X_out, w.Wq, w.s_w, w.W_out,
                             None if flags_null else q.flags, Y, status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        o = oracle_layer(X, W, idx, "w8", synth.THRESHOLD)
        assert_y_close(Y.cpu().numpy(), o["y"], f"flags null {flags_null}")


# ------------------------------------------------------------ 4-bit weights
@pytest.mark.parametrize("M,N,K", [(256, 256, 128), (512, 512, 1024), (300, 384, 512),
                                   (1000, 1280, 2048), (2048, 4096, 1024), (257, 4992, 256),
                                   (200, 256, 384), (2048, 8192, 640), (2304, 8064, 384)])
def test_pair_w4_int32_bit_exact(gpu, M, N, K):
    # (2048, 8192, 640): three jobs per tile (an odd count) over several tiles
    # per pair, so consecutive tiles start on jobs of either expansion group
    # and on any shared-memory slot; (2304, 8064, 384): a one-block last job,
    # and N % 256 == 128 (the second CTA's rows of the last column tile absent)
    torch, mq = gpu.torch, gpu.mq
    W = synth.weights(N, K, seed=M + N + 1)
    w = mq.prepack(gpu.dev(W), gpu.dev(np.zeros(0, np.int32)), mq.MIXQ_W4G128)
    Wq8, _, _ = oracle.prepack_w8(W, [])
    w8eff = oracle.prepack_w4(Wq8)[3]
    Xq = np.random.default_rng(M * 5 + K).integers(-127, 128, size=(M, K)).astype(np.int8)
    acc = gpu.acc_i32(Xq, w, bn=512)
    rows = (0, M) if M * N * K <= 2 ** 31 else (M // 2 - 8, M // 2 + 8)
    np.testing.assert_array_equal(acc[rows[0]:rows[1]], oracle.gemm_i32(Xq, w8eff, *rows))
    if rows != (0, M):
        np.testing.assert_array_equal(acc[M - 8:], oracle.gemm_i32(Xq, w8eff, M - 8, M))


def test_pair_w4_int32_matches_the_tensor_memory_kernel(gpu):
    M, N, K = 1536, 11008, 4096
    W = synth.weights(N, K)
    torch, mq = gpu.torch, gpu.mq
    w = mq.prepack(gpu.dev(W), gpu.dev(np.zeros(0, np.int32)), mq.MIXQ_W4G128)
    Xq = gpu.dev(np.random.default_rng(4).integers(-127, 128, size=(M, K)).astype(np.int8))
    np.testing.assert_array_equal(gpu.acc_i32(Xq, w, bn=512), gpu.acc_i32(Xq, w, bn=256))


@pytest.mark.parametrize("M,N,K,k_out", [(2048, 5120, 1024, 64), (2304, 4992, 2048, 256),
                                         (2048, 5120, 1024, 0), (2048, 11008, 4096, 128),
                                         (2100, 640, 384, 32), (4096, 4096, 4096, 256),
                                         (2048, 8192, 640, 128), (2560, 6144, 1152, 128)])
def test_pair_w4_layer_within_tolerance(gpu, M, N, K, k_out):
    # the last two: odd job counts per tile (3 INT8 + 2 outlier jobs; 5 + 2)
    # over several tiles per pair
    mq = gpu.mq
    assert mq.mixq_gemm_plan(mq.MIXQ_W4G128, M, N, K)[0] == 256
    idx = synth.outlier_channels(K, k_out)
    X = synth.activations(M, K, idx, synth.channel_factors(k_out)) if k_out else \
        synth.activations(M, K)
    W = synth.weights(N, K)
    g = gpu.layer(X, W, idx, "w4", synth.THRESHOLD)
    assert g["status"] == 0
    rows = (0, M) if M * N * K <= 2 ** 33 else (M // 2 - 6, M // 2 + 6)
    o = oracle_layer(X, W, idx, "w4", synth.THRESHOLD, rows)
    assert_y_close(g["Y"][rows[0]:rows[1]], o["y"], f"pair w4 M{M} N{N} K{K} ko{k_out}")
    if rows != (0, M):
        o2 = oracle_layer(X, W, idx, "w4", synth.THRESHOLD, (M - 4, M))
        assert_y_close(g["Y"][M - 4:], o2["y"], "last rows")
