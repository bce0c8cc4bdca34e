"""Randomised invariants of the oracle (no GPU): symmetries and error bounds that
any correct implementation of the definitions has, checked on inputs drawn by
hypothesis (derandomized, no example database, bounded example counts)."""
import numpy as np
from hypothesis import HealthCheck, assume, given, settings
from hypothesis import strategies as st

import oracle

SETTINGS = dict(max_examples=40, deadline=None, derandomize=True, database=None,
                suppress_health_check=[HealthCheck.too_slow])


def _acts(seed, M, K, k_out, scale):
    rng = np.random.default_rng(seed)
    X = (rng.standard_normal((M, K)) * scale).astype(np.float16)
    idx = np.sort(rng.choice(K, k_out, replace=False)).astype(np.int32)
    X[:, idx] *= np.float16(rng.uniform(1, 40))
    return X, idx


@settings(**SETTINGS)
@given(seed=st.integers(0, 2**31 - 1), M=st.integers(1, 9), kb=st.integers(1, 3),
       k_out=st.integers(0, 12), T=st.sampled_from([0.5, 3.0, 6.0, 40.0]))
def test_token_permutation_and_round_trip(seed, M, kb, k_out, T):
    """Permuting tokens permutes every per-token output and leaves the detection
    outputs alone; every quantized element is within half a step of its value
    (plus the fp32 rounding of the scale arithmetic)."""
    K = 128 * kb
    X, idx = _acts(seed, M, K, k_out, 2.0)
    Xq, s_x, X_out, bitmap, flags = oracle.quantize_act(X, idx, T)
    perm = np.random.default_rng(seed + 1).permutation(M)
    Xq2, s_x2, X_out2, bitmap2, flags2 = oracle.quantize_act(X[perm], idx, T)
    np.testing.assert_array_equal(Xq2, Xq[perm])
    np.testing.assert_array_equal(s_x2, s_x[perm])
    np.testing.assert_array_equal(X_out2.view(np.uint16), X_out[perm].view(np.uint16))
    np.testing.assert_array_equal(bitmap2, bitmap)
    np.testing.assert_array_equal(flags2, flags)
    x = X.astype(np.float64)
    in_idx = np.zeros(K, bool)
    in_idx[idx] = True
    mixed = (k_out > 0) & (np.abs(x).max(axis=1) > T)
    assert flags[0] == mixed.sum()
    keep = ~(mixed[:, None] & in_idx[None, :])  # elements that stay in the INT8 part
    # half a step, plus the three fp32 roundings of 127/a, x*(127/a) and a/127:
    # |x| <= a = 127 s, so they add at most 127 s * 3 * 2^-24 < 3e-5 s
    err = np.abs(x - s_x.astype(np.float64)[:, None] * Xq)
    bound = np.broadcast_to(s_x.astype(np.float64)[:, None] * (0.5 + 3e-5), err.shape)
    assert (err[keep] <= bound[keep]).all()
    assert not Xq[~keep].any()
    assert np.abs(Xq.astype(np.int32)).max(initial=0) <= 127


@settings(**SETTINGS)
@given(seed=st.integers(0, 2**31 - 1), M=st.integers(1, 6), e=st.integers(-3, 3))
def test_power_of_two_scaling(seed, M, e):
    """With no outlier list, scaling a token by 2^e scales s_x by 2^e and keeps the
    codes; scaling a weight row by 2^e does the same for s_w and Wq."""
    K = 256
    X, _ = _acts(seed, M, K, 0, 1.0)
    f = np.float16(2.0 ** e)
    assume((X.astype(np.float64) * float(f) == (X * f).astype(np.float64)).all())  # exact in fp16
    Xq, s_x, _, _, _ = oracle.quantize_act(X, [], 1e9)
    Xq2, s_x2, _, _, _ = oracle.quantize_act(X * f, [], 1e9)
    np.testing.assert_array_equal(Xq2, Xq)
    np.testing.assert_array_equal(s_x2, s_x * np.float32(f))
    W = X  # any fp16 matrix serves as weights
    Wq, s_w, _ = oracle.prepack_w8(W, [])
    Wq2, s_w2, _ = oracle.prepack_w8(W * f, [])
    np.testing.assert_array_equal(Wq2, Wq)
    np.testing.assert_array_equal(s_w2, s_w * np.float32(f))


@settings(**SETTINGS)
@given(seed=st.integers(0, 2**31 - 1), N=st.integers(1, 6), M=st.integers(1, 5),
       kb=st.integers(1, 3))
def test_layer_rows_and_columns_are_independent(seed, N, M, kb):
    """Output [m, n] depends only on token m and weight row n: a window of rows and
    a permutation of weight rows give the matching slice and permutation of y, for
    both weight formats of the layer."""
    K = 128 * kb
    X, idx = _acts(seed, M, K, 3, 1.0)
    W = (np.random.default_rng(seed + 2).standard_normal((N, K)) * 0.02).astype(np.float16)
    Xq, s_x, X_out, _, _ = oracle.quantize_act(X, idx, 6.0)
    Wq, s_w, W_out = oracle.prepack_w8(W, idx)
    perm = np.random.default_rng(seed + 3).permutation(N)
    acc, y = oracle.linear(Xq, s_x, X_out, Wq, s_w, W_out)
    acc2, y2 = oracle.linear(Xq, s_x, X_out, Wq[perm], s_w[perm], W_out[perm])
    np.testing.assert_array_equal(acc2, acc[:, perm])
    np.testing.assert_array_equal(y2, y[:, perm])
    m0 = M // 2
    acc3, y3 = oracle.linear(Xq, s_x, X_out, Wq, s_w, W_out, m0, M)
    np.testing.assert_array_equal(acc3, acc[m0:])
    np.testing.assert_array_equal(y3, y[m0:])
    q, s_g, z_g = oracle.prepack_w4b(W)
    q2, s_g2, z_g2 = oracle.prepack_w4b(W[perm])
    np.testing.assert_array_equal(q2, q[perm])
    part, yb = oracle.linear_w4b(Xq, s_x, X_out, q, s_g, z_g, W_out)
    part2, yb2 = oracle.linear_w4b(Xq, s_x, X_out, q2, s_g2, z_g2, W_out[perm])
    np.testing.assert_array_equal(part2, part[:, perm])
    np.testing.assert_array_equal(yb2, yb[:, perm])


@settings(**SETTINGS)
@given(seed=st.integers(0, 2**31 - 1), e=st.integers(-10, 2), ng=st.integers(1, 4))
def test_w4b_planted_codes_any_scale(seed, e, ng):
    """Weights s0 (q - z) with q spanning 0..15 in every group come back exactly,
    for power-of-two scales across the normal fp16 range."""
    rng = np.random.default_rng(seed)
    N, K = 3, 128 * ng
    z0 = rng.integers(0, 16, size=(N, ng))
    q0 = rng.integers(0, 16, size=(N, ng, 128))
    q0[:, :, 0], q0[:, :, 1] = 0, 15
    s0 = 2.0 ** e
    W = (s0 * (q0 - z0[:, :, None])).reshape(N, K).astype(np.float16)
    q, s_g, z_g = oracle.prepack_w4b(W)
    np.testing.assert_array_equal(q, q0.reshape(N, K))
    np.testing.assert_array_equal(z_g, z0)
    assert (s_g.astype(np.float64) == s0).all()
