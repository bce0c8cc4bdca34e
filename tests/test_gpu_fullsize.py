"""Full-size workloads (the Llama-7B decode and prefill shapes, the W4A8
variant, the Llama-70B batch-512 shapes) through the same launch path the
benchmark times, checked against the oracle: every quantized code, scale,
gathered outlier value, bitmap bit and flag bit for bit over the whole
matrices, and the FP16 layer output at sampled (token, channel) points that
the oracle computes one by one (plus every output of the first and last
token)."""
import functools

import numpy as np
import pytest

import oracle
import synth
from helpers import Gpu, assert_y_close

pytestmark = pytest.mark.gpu

CASES = (synth.decode("w8") + synth.decode("w4") + synth.prefill("w8") + synth.prefill("w4")
         + synth.llama70b("w8") + synth.llama70b("w4"))


@pytest.fixture(scope="module")
def gpu():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    return Gpu()


@functools.lru_cache(maxsize=2)
def _weights(N, K):
    return synth.weights(N, K)


@functools.lru_cache(maxsize=4)
def _oracle_weights(N, K, k_out, mode):
    W = _weights(N, K)
    idx = synth.outlier_channels(K, k_out)
    Wq8, s_w, W_out = oracle.prepack_w8(W, idx)
    if mode == "w8":
        return Wq8, s_w, W_out, None
    q, s2, z2, w8 = oracle.prepack_w4(Wq8)
    return w8, s_w, W_out, (q, s2, z2)


@pytest.mark.parametrize("case", CASES, ids=lambda c: c.name)
def test_full_size_case(gpu, case):
    idx = case.channels()
    if case.scaled and case.k_out:
        f = case.factor if case.factor is not None else synth.channel_factors(case.k_out)
        X = synth.activations(case.M, case.K, idx, f)
    else:
        X = synth.activations(case.M, case.K)
    W = _weights(case.N, case.K)
    g = gpu.layer(X, W, idx, case.mode, case.threshold)
    assert g["status"] == 0
    Xq, s_x, X_out, bitmap, flags = oracle.quantize_act(X, idx, case.threshold)
    np.testing.assert_array_equal(g["Xq"], Xq)
    np.testing.assert_array_equal(g["s_x"].view(np.uint32), s_x.view(np.uint32))
    np.testing.assert_array_equal(g["X_out"].view(np.uint16), X_out.view(np.uint16))
    np.testing.assert_array_equal(g["bitmap"], bitmap)
    assert list(g["flags"]) == [flags[0], flags[1], 0, 0]
    Weff, s_w, W_out, w4 = _oracle_weights(case.N, case.K, case.k_out, case.mode)
    np.testing.assert_array_equal(g["s_w"].view(np.uint32), s_w.view(np.uint32))
    np.testing.assert_array_equal(g["W_out"].view(np.uint16), W_out.view(np.uint16))
    if case.mode == "w8":
        np.testing.assert_array_equal(g["Wq"], Weff)
    else:
        q, s2, z2 = gpu.unpack_w4(g["packed"])
        np.testing.assert_array_equal(q, w4[0])
        np.testing.assert_array_equal(s2, w4[1])
        np.testing.assert_array_equal(z2, w4[2])
    rng = np.random.default_rng(1234)
    P = 4096
    ms = np.concatenate([rng.integers(0, case.M, P), np.zeros(case.N, np.int64),
                         np.full(case.N, case.M - 1)]).astype(np.int32)
    ns = np.concatenate([rng.integers(0, case.N, P), np.arange(case.N),
                         np.arange(case.N)]).astype(np.int32)
    xo = X_out if X_out.shape[1] else None
    wo = W_out if W_out.shape[1] else None
    _, y = oracle.linear_points(Xq, s_x, xo, Weff, s_w, wo, ms, ns)
    assert_y_close(g["Y"][ms, ns], y, case.name)
