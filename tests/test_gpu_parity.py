"""CUDA path vs the CPU oracle, through the C ABI (needs a B200).

Codes, scales, gathered outlier matrices, detection bitmaps, flags and INT32
accumulators must match bit for bit; the FP16 layer output must satisfy
|Y - y| <= max(1e-3, 1e-2 |y|) against the oracle's fp64 value.
"""
import functools
import json
import os

import numpy as np
import pytest

import oracle
import synth
from helpers import Gpu, assert_y_close, oracle_layer, oracle_weights

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gpu():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    return Gpu()


def _assert_quant_equal(g, o, what):
    np.testing.assert_array_equal(g["Xq"], o["Xq"], err_msg=f"{what}: Xq")
    np.testing.assert_array_equal(g["s_x"].view(np.uint32), o["s_x"].view(np.uint32),
                                  err_msg=f"{what}: s_x")
    np.testing.assert_array_equal(g["X_out"].view(np.uint16), o["X_out"].view(np.uint16),
                                  err_msg=f"{what}: X_out")
    np.testing.assert_array_equal(g["bitmap"], o["bitmap"], err_msg=f"{what}: bitmap")
    assert list(g["flags"][:2]) == list(o["flags"]), (what, g["flags"], o["flags"])
    assert list(g["flags"][2:]) == [0, 0], (what, g["flags"])


def _assert_weights_equal(gpu, g, o, mode, what):
    np.testing.assert_array_equal(g["s_w"].view(np.uint32), o["s_w"].view(np.uint32),
                                  err_msg=f"{what}: s_w")
    np.testing.assert_array_equal(g["W_out"].view(np.uint16), o["W_out"].view(np.uint16),
                                  err_msg=f"{what}: W_out")
    if mode == "w8":
        np.testing.assert_array_equal(g["Wq"], o["Wq8"], err_msg=f"{what}: Wq")
    else:
        q, s2, z2 = gpu.unpack_w4(g["packed"])
        np.testing.assert_array_equal(q, o["q"], err_msg=f"{what}: q")
        np.testing.assert_array_equal(s2, o["s2"], err_msg=f"{what}: s2")
        np.testing.assert_array_equal(z2, o["z2"], err_msg=f"{what}: z2")


# ------------------------------------------------------------ tiny workload
@pytest.mark.parametrize("mode", ["w8", "w4"])
def test_tiny_layer_bit_exact_and_within_tolerance(gpu, mode):
    (case,) = synth.tiny()
    X, W, idx = case.make()
    g = gpu.layer(X, W, idx, mode, case.threshold)
    o = oracle_layer(X, W, idx, mode, case.threshold)
    assert g["status"] == 0
    _assert_quant_equal(g, o, "tiny")
    _assert_weights_equal(gpu, g, o, mode, "tiny")
    detected = [k for k in range(case.K) if g["bitmap"][k // 32] >> (k % 32) & 1]
    assert detected == [3, 77, 130, 201]
    assert g["flags"][0] == case.M
    assert_y_close(g["Y"], o["y"], "tiny Y")


# ---------------------------------------------------- quantize edge cases
def _golden_sets():
    path = os.path.join(os.path.dirname(__file__), "golden", "quantize_cases.json")
    with open(path) as f:
        return json.load(f)["sets"]


@pytest.mark.parametrize("gset", _golden_sets(), ids=lambda s: s["name"])
def test_quantize_golden_cases_on_gpu(gpu, gset):
    K = 128  # the golden rows (K=64) padded with zero channels to the ABI's K multiple
    X = np.zeros((len(gset["rows"]), K), np.float16)
    for m, r in enumerate(gset["rows"]):
        for k, v in r["x"].items():
            X[m, int(k)] = v
    idx = np.asarray(gset["idx"], np.int32)
    W = synth.weights(128, K)
    g = gpu.layer(X, W, idx, "w8", gset["T"])
    o = oracle_layer(X, W, idx, "w8", gset["T"])
    _assert_quant_equal(g, o, gset["name"])
    assert list(g["flags"][:2]) == gset["flags"]
    assert_y_close(g["Y"], o["y"], gset["name"])


@pytest.mark.parametrize("M,K,k_out", [(1, 128, 0), (1, 256, 1), (3, 384, 5), (129, 512, 64),
                                       (300, 1024, 130), (5, 256, 256), (2, 28672, 64),
                                       (33, 4096, 64), (24, 8192, 64), (64, 11008, 64),
                                       (48, 12288, 100)])
def test_quantize_shapes(gpu, M, K, k_out):
    idx = synth.outlier_channels(K, k_out)
    X = synth.activations(M, K, idx, synth.channel_factors(k_out)) if k_out else \
        synth.activations(M, K, [7], [30.0])
    W = synth.weights(128, K)
    g = gpu.layer(X, W, idx, "w8", 6.0)
    o = oracle_layer(X, W, idx, "w8", 6.0)
    _assert_quant_equal(g, o, f"M{M} K{K} ko{k_out}")
    assert_y_close(g["Y"], o["y"], f"M{M} K{K} ko{k_out}")


def test_threshold_boundaries(gpu):
    K = 256
    X = np.zeros((4, K), np.float16)
    X[:, 10] = 0.5
    X[0, 3] = 6.0
    X[1, 3] = np.nextafter(np.float16(6.0), np.float16(np.inf))
    X[2, 64] = -7.0
    X[3, 100] = 6.0
    idx = np.array([3, 64], np.int32)
    W = synth.weights(128, K)
    g = gpu.layer(X, W, idx, "w8", 6.0)
    o = oracle_layer(X, W, idx, "w8", 6.0)
    _assert_quant_equal(g, o, "threshold")
    assert g["flags"][0] == 2


def test_bad_idx_reported_on_device(gpu):
    import torch
    mq = gpu.mq
    X = gpu.dev(synth.activations(4, 256))
    idx = gpu.dev(np.array([9, 3], np.int32))  # not sorted
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    mq.quantize_act(X, idx, 6.0, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 1


@pytest.mark.parametrize("T", [6.0, 6.001, 5.9990234375, 0.3, 1e5])
@pytest.mark.parametrize("M,K", [(3, 512), (40, 2048), (300, 4096)])
def test_quantize_threshold_between_fp16_values(gpu, T, M, K):
    """The outlier test |x| > T with T not an fp16 value: activations placed on
    the fp16 neighbours of T (and their negatives) in outlier and ordinary
    channels; codes, scales, X_out, bitmap and flags bit for bit."""
    rng = np.random.default_rng(int(T * 1000) % 97 + M)
    X = (rng.standard_normal((M, K)) * 0.3).astype(np.float16)
    t = np.float16(T) if np.isfinite(np.float16(T)) else np.float16(65504)
    below = t if float(t) <= T else np.nextafter(t, np.float16(-np.inf))
    with np.errstate(over="ignore"):
        neigh = [below, np.nextafter(below, np.float16(np.inf)),
                 np.nextafter(below, np.float16(-np.inf))]
    neigh = [n if np.isfinite(n) else np.float16(65504) for n in neigh]
    idx = synth.outlier_channels(K, 16)
    cols = [int(idx[1]), int(idx[5]), 7, 300, K - 1]
    for j, c in enumerate(cols):
        for r in range(0, M, 3):
            v = neigh[(j + r) % 3]
            X[r, c] = v if (r + j) % 2 == 0 else -v
    W = synth.weights(128, K)
    g = gpu.layer(X, W, idx, "w8", T)
    o = oracle_layer(X, W, idx, "w8", T)
    assert g["status"] == 0
    _assert_quant_equal(g, o, f"T={T} M{M} K{K}")


# ---------------------------------------------------------- INT32 mainloop
@functools.lru_cache(maxsize=None)
def _packed_random(N, K, mode_i):
    """Random fp16 weights prepacked by the oracle (host) -- returns oracle data."""
    W = synth.weights(N, K, seed=100 + K + N)
    Weff, _, _, extra = oracle_weights(W, [], "w8" if mode_i == 0 else "w4")
    return W, Weff


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("M,N,K", [(1, 128, 128), (3, 256, 256), (130, 384, 512), (200, 256, 1024),
                                   (64, 512, 4096), (257, 128, 384), (1100, 256, 512)])
@pytest.mark.parametrize("bn,split", [(0, 0), (0, 2), (128, 1), (256, 1), (256, 2), (128, 4),
                                      (256, 8), (32, 1), (64, 3), (32, 8)])
def test_int32_accumulators_bit_exact(gpu, mode, M, N, K, bn, split):
    if split > K // 128:
        pytest.skip("split larger than the number of K blocks")
    if bn < 128 and M > 64:
        pytest.skip("narrow tiles are for M <= 64")
    if mode == 1 and bn == 128 and split > 1 and M > 64:
        pytest.skip("the two-CTA W4 variant splits K only for M <= 64")
    if mode == 1 and bn == 256 and split > 1 and M > 1024:
        pytest.skip("the one-CTA W4 variant splits K only for M <= 1024")
    import torch
    rng = np.random.default_rng(M * 7 + N + K)
    Xq = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    W, Weff = _packed_random(N, K, mode)
    w = gpu.mq.prepack(gpu.dev(W), torch.zeros(0, dtype=torch.int32, device="cuda"), mode)
    acc = gpu.acc_i32(Xq, w, bn, split)
    np.testing.assert_array_equal(acc, oracle.gemm_i32(Xq, Weff))


# ------------------------------------------------------------- layer output
@pytest.mark.parametrize("mode", ["w8", "w4"])
@pytest.mark.parametrize("M,K,N,k_out", [(16, 512, 256, 4), (64, 1024, 640, 64), (130, 512, 384, 1),
                                         (260, 768, 512, 130), (8, 1024, 1024, 0),
                                         (1, 2048, 512, 64), (24, 1024, 512, 16),
                                         (40, 2048, 384, 32)])
def test_layer_output_within_tolerance(gpu, mode, M, K, N, k_out):
    idx = synth.outlier_channels(K, k_out)
    X = synth.activations(M, K, idx, synth.channel_factors(k_out)) if k_out else \
        synth.activations(M, K)
    W = synth.weights(N, K)
    g = gpu.layer(X, W, idx, mode, 6.0)
    o = oracle_layer(X, W, idx, mode, 6.0)
    _assert_quant_equal(g, o, "layer")
    _assert_weights_equal(gpu, g, o, mode, "layer")
    assert_y_close(g["Y"], o["y"], f"{mode} M{M} K{K} N{N} ko{k_out}")


@pytest.mark.parametrize("mode", ["w8", "w4"])
def test_fast_path_no_token_mixed(gpu, mode):
    """Unscaled activations: no token exceeds T, the fp16 slice is skipped and the
    layer is the plain W8A8 (or W4A8) product."""
    M, K, N = 64, 1024, 512
    idx = synth.outlier_channels(K, 64)
    X = synth.activations(M, K)
    W = synth.weights(N, K)
    g = gpu.layer(X, W, idx, mode, 6.0)
    o = oracle_layer(X, W, idx, mode, 6.0)
    assert o["flags"][0] == 0 and g["flags"][0] == 0
    _assert_quant_equal(g, o, "fast path")
    assert_y_close(g["Y"], o["y"], "fast path")


def test_every_channel_an_outlier(gpu):
    """idx = all K, every token mixed: the INT8 part is zero and Y is the fp16 product."""
    M, K, N = 32, 256, 256
    X = synth.activations(M, K)
    X[:, 1] = 8.0
    W = synth.weights(N, K)
    idx = np.arange(K, dtype=np.int32)
    g = gpu.layer(X, W, idx, "w8", 6.0)
    assert not g["Xq"].any() and g["flags"][0] == M
    ref = X.astype(np.float64) @ W.astype(np.float64).T
    assert_y_close(g["Y"], ref, "all-outlier")


# --------------------------------------------------- stall -> timeout status
def test_stalled_pipeline_times_out_with_status(gpu):
    import torch
    mq = gpu.mq
    M, K, N = 128, 256, 256
    Xq = torch.zeros((M, K), dtype=torch.int8, device="cuda")
    Wq = torch.zeros((N, K), dtype=torch.int8, device="cuda")
    s = torch.ones(max(M, N), dtype=torch.float32, device="cuda")
    Y = torch.zeros((M, N), dtype=torch.float16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    mq.mixq_debug_gemm_stall(Xq, Wq, s, s, Y, 20_000_000, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 5
    # the context is still usable: a normal layer runs and matches the oracle
    (case,) = synth.tiny()
    X, W, idx = case.make()
    g = gpu.layer(X, W, idx, "w8", case.threshold)
    o = oracle_layer(X, W, idx, "w8", case.threshold)
    assert_y_close(g["Y"], o["y"], "after stall")


def test_host_errors_are_synchronous(gpu):
    import torch
    mq = gpu.mq
    Xq = torch.zeros((4, 256), dtype=torch.int8, device="cuda")
    rc = mq.lib().mixq_gemm_w8a8o16(4, 200, 256, 0, Xq.data_ptr(), 0, 0, 0, 0, 0, 0, 0, 256, 0, 0)
    assert rc == 2
    rc = mq.lib().mixq_gemm_w8a8o16(4, 256, 256, 0, Xq.data_ptr() + 1, Xq.data_ptr(), 0,
                                    Xq.data_ptr(), Xq.data_ptr(), 0, 0, Xq.data_ptr(), 256, 0, 0)
    assert rc == 3
