"""Pins for the CPU oracle (no GPU).

The oracle is checked against facts that do not come from the oracle itself:
hand-derived closed-form cases (tests/golden), exact integer arithmetic done a
different way (pure-Python brute force, numpy int64/fp64 products), invariants
that reduce the layer to a simpler textbook computation (no outliers -> plain
W8A8; every channel an outlier -> the plain fp16 product), a rigorous
quantization error bound against the exact fp64 product, and exhaustive checks
of the 4-bit level-2 rules (range, no-overflow, round-trip bound), and the
same kinds of checks for the 4-bit reading-B weights (planted codes, round
trip, dense-product equivalence).
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synth


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


def _row(K, entries):
    x = np.zeros(K, np.float16)
    for k, v in entries.items():
        x[int(k)] = np.float16(v)
    return x


def _f32_ratio(pair):
    return np.float32(pair[0]) / np.float32(pair[1])


# ---------------------------------------------------------------- activations

def test_quantize_golden_cases(golden_dir):
    g = _load(golden_dir, "quantize_cases.json")
    for s in g["sets"]:
        K, idx, T = s["K"], s["idx"], s["T"]
        X = np.stack([_row(K, r["x"]) for r in s["rows"]])
        Xq, s_x, X_out, bitmap, flags = oracle.quantize_act(X, idx, T)
        for m, r in enumerate(s["rows"]):
            want = np.zeros(K, np.int8)
            for k, v in r["codes"].items():
                want[int(k)] = v
            np.testing.assert_array_equal(Xq[m], want, err_msg=f"{s['name']} row {m}: {r['why']}")
            assert s_x[m] == _f32_ratio(r["s_x"]), (s["name"], m)
            if "x_out" in r:
                np.testing.assert_array_equal(X_out[m, : len(idx)], np.float16(r["x_out"]))
                assert not X_out[m, len(idx):].any()
        want_bits = np.zeros((K + 31) // 32, np.uint32)
        for k in s["bitmap_channels"]:
            want_bits[k // 32] |= np.uint32(1 << (k % 32))
        np.testing.assert_array_equal(bitmap, want_bits)
        assert list(flags) == s["flags"]


def test_threshold_strict_and_abs():
    """x = T is not an outlier, the next fp16 above T is, and so is -T-1."""
    K, T = 128, 6.0
    idx = [3, 64]
    X = np.zeros((4, K), np.float16)
    X[0, 3] = 6.0
    X[1, 3] = np.nextafter(np.float16(6.0), np.float16(np.inf))
    X[2, 64] = -7.0
    X[3, 100] = 6.0
    _, _, X_out, bitmap, flags = oracle.quantize_act(X, idx, T)
    assert flags[0] == 2
    assert flags[1] == 0
    assert bitmap[0] == 1 << 3 and bitmap[2] == 1 and bitmap[1] == 0 and bitmap[3] == 0
    assert X_out[1, 0] == X[1, 3] and X_out[2, 1] == -7.0
    assert not X_out[0].any() and not X_out[3].any()


def test_kout_zero_never_mixed():
    X = synth.activations(8, 256, [5], [100.0])
    Xq, s_x, X_out, bitmap, flags = oracle.quantize_act(X, [], 6.0)
    assert flags[0] == 0 and X_out.shape[1] == 0
    assert bitmap[0] == 1 << 5 and flags[1] == 1
    # the outlier channel stays in INT8 and sets the scale
    assert (np.abs(Xq[:, 5]) == 127).all()


def test_kout_all_channels():
    """idx = all K and every token mixed: Xq == 0, X_out == X."""
    M, K = 5, 128
    X = synth.activations(M, K)
    X[:, 7] = 10.0
    idx = np.arange(K, dtype=np.int32)
    Xq, s_x, X_out, bitmap, flags = oracle.quantize_act(X, idx, 6.0)
    assert flags[0] == M and flags[1] == 0
    assert not Xq.any() and not s_x.any()
    np.testing.assert_array_equal(X_out[:, :K].view(np.uint16), X.view(np.uint16))


def test_tiny_detects_exactly_the_four_channels():
    (case,) = synth.tiny()
    X, W, idx = case.make()
    _, _, _, bitmap, flags = oracle.quantize_act(X, idx, case.threshold)
    got = [k for k in range(case.K) if bitmap[k // 32] >> (k % 32) & 1]
    assert got == [3, 77, 130, 201]
    assert flags[0] == case.M and flags[1] == 0


def test_invalid_idx_rejected():
    X = np.zeros((2, 64), np.float16)
    for bad in ([5, 5], [7, 3], [-1], [64]):
        with pytest.raises(oracle.OracleError):
            oracle.quantize_act(X, bad, 6.0)


def test_nonfinite_rejected():
    X = np.zeros((2, 64), np.float16)
    X[1, 3] = np.inf
    with pytest.raises(oracle.OracleError):
        oracle.quantize_act(X, [], 6.0)


# ------------------------------------------------------------------- weights

def test_prepack_w8_closed_form():
    """Row amax 127 -> s_w = 1 and codes = rint(w); amax over ALL columns."""
    K = 128
    W = np.zeros((3, K), np.float16)
    W[0, :4] = [127.0, -0.5, 1.5, -2.5]
    W[1, 10] = -2.0          # a = 2 -> s = 2/127, inv = 63.5
    W[1, 11] = 1.0
    W[2, 5] = 100.0          # outlier column carries the row max: still part of the range
    W[2, 6] = 50.0
    Wq, s_w, W_out = oracle.prepack_w8(W, [5, 11])
    np.testing.assert_array_equal(Wq[0, :4], [127, 0, 2, -2])
    assert s_w[0] == np.float32(1.0)
    assert Wq[1, 10] == -127 and Wq[1, 11] == 64 and s_w[1] == np.float32(2) / np.float32(127)
    assert Wq[2, 5] == 127 and Wq[2, 6] == 64 and s_w[2] == np.float32(100) / np.float32(127)
    np.testing.assert_array_equal(W_out[:, 0], W[:, 5])
    np.testing.assert_array_equal(W_out[:, 1], W[:, 11])
    assert W_out.shape == (3, 64) and not W_out[:, 2:].any()


def test_w4_golden_cases(golden_dir):
    g = _load(golden_dir, "w4_level2_cases.json")
    for c in g["cases"]:
        row = np.full(128, c["lo"], np.int8)
        row[1] = c["hi"]
        vals = [p[0] for p in c["pairs"]]
        row[2: 2 + len(vals)] = vals
        q, s2, z2, w8 = oracle.prepack_w4(row[None, :])
        assert s2[0, 0] == c["s2"] and z2[0, 0] == c["z2"], c["why"]
        for i, (w, qq, eff) in enumerate(c["pairs"]):
            assert q[0, 2 + i] == qq and w8[0, 2 + i] == eff, (c["why"], w)


def test_w4_exhaustive_invariants():
    """Every (lo, hi) range: q in [0,15], w8eff in int8, byte-parallel no-overflow
    (q*s2 <= 255, z2*s2 <= 255), and |w8eff - w8| <= s2/2 unless clamped."""
    rows = []
    for lo in range(-127, 128, 3):
        for hi in range(lo, 128, 5):
            r = np.linspace(lo, hi, 128).round().astype(np.int8)
            r[0], r[-1] = lo, hi
            rows.append(r)
    W8 = np.stack(rows)
    q, s2, z2, w8 = oracle.prepack_w4(W8)
    s = s2[:, :1].astype(np.int32)
    z = z2[:, :1].astype(np.int32)
    assert q.max() <= 15
    assert (s >= 1).all() and (s <= 17).all() and (z <= 15).all()
    assert (q.astype(np.int32) * s).max() <= 255 and (z * s).max() <= 255
    lo = W8.min(axis=1, keepdims=True).astype(np.int32)
    hi = W8.max(axis=1, keepdims=True).astype(np.int32)
    assert ((hi - lo) <= 15 * s).all() and ((s == 1) | ((hi - lo) > 15 * (s - 1))).all()
    np.testing.assert_array_equal(w8.astype(np.int32), (q.astype(np.int32) - z) * s)
    # groups whose range straddles zero: a clamp moves a code by at most one
    # step (error <= 1.5*s2); codes strictly inside the group's code range are
    # unclamped and round to the nearest multiple of s2 (error <= s2/2)
    ok = ((lo <= 0) & (hi >= 0)).reshape(-1)
    err = np.abs(w8.astype(np.int32) - W8.astype(np.int32))[ok]
    qq = q[ok].astype(np.int32)
    inner = (qq > qq.min(axis=1, keepdims=True)) & (qq < qq.max(axis=1, keepdims=True))
    assert (2 * err <= 3 * s[ok]).all()
    assert (2 * err <= s[ok])[inner].all()
    assert inner.sum() > 0.8 * inner.size


def test_w4_unit_scale_special_case_is_exact():
    """Every group spans <= 16 consecutive integers inside [-15, 15] -> s2 = 1 and
    w8eff == w8, so the W4A8 product equals the W8A8 product exactly."""
    rng = np.random.default_rng(11)
    N, K = 6, 512
    lo = rng.integers(-15, 1, size=(N, K // 128, 1))
    W8 = (lo + rng.integers(0, 16, size=(N, K // 128, 128))).clip(-127, 127).reshape(N, K)
    W8 = W8.astype(np.int8)
    q, s2, z2, w8 = oracle.prepack_w4(W8)
    assert (s2 == 1).all()
    np.testing.assert_array_equal(w8, W8)
    Xq = rng.integers(-127, 128, size=(4, K)).astype(np.int8)
    np.testing.assert_array_equal(oracle.gemm_i32(Xq, w8), oracle.gemm_i32(Xq, W8))


def test_fp32_division_rounding_matches_exact_rational():
    """rint(w8/s2) in fp32 equals exact half-even rounding of the rational w8/s2."""
    for s in range(1, 18):
        for w in range(-128, 128):
            f = Fraction(w, s)
            fl = int(np.floor(float(f)))
            frac = f - fl
            exact = fl + (1 if frac > Fraction(1, 2) or (frac == Fraction(1, 2) and fl % 2) else 0)
            assert int(np.rint(np.float32(w) / np.float32(s))) == exact


# -------------------------------------------------------------------- GEMM

def test_gemm_int32_brute_force_tiny():
    rng = np.random.default_rng(5)
    for M, N, K in ((1, 1, 128), (3, 5, 128), (8, 8, 256), (7, 2, 256)):
        Xq = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
        Wq = rng.integers(-128, 128, size=(N, K)).astype(np.int8)
        Xq[0, :3] = [127, -127, 127]
        acc = oracle.gemm_i32(Xq, Wq)
        for m in range(M):
            for n in range(N):
                assert acc[m, n] == sum(int(Xq[m, k]) * int(Wq[n, k]) for k in range(K))
        np.testing.assert_array_equal(acc, Xq.astype(np.int64) @ Wq.astype(np.int64).T)
        np.testing.assert_array_equal(acc, (Xq.astype(np.float64) @ Wq.astype(np.float64).T))


def test_gemm_int32_extremes_fit():
    """Largest K of the workloads with extreme codes stays inside int32."""
    K = 28672
    Xq = np.full((2, K), -127, np.int8)
    Xq[1] = 127
    Wq = np.full((2, K), -128, np.int8)
    Wq[1] = 127
    acc = oracle.gemm_i32(Xq, Wq)
    assert acc[0, 0] == 127 * 128 * K and acc[1, 1] == 127 * 127 * K
    assert acc[0, 1] == -127 * 127 * K


def test_gemm_row_window():
    rng = np.random.default_rng(6)
    Xq = rng.integers(-127, 128, size=(9, 256)).astype(np.int8)
    Wq = rng.integers(-127, 128, size=(4, 256)).astype(np.int8)
    full = oracle.gemm_i32(Xq, Wq)
    np.testing.assert_array_equal(oracle.gemm_i32(Xq, Wq, 3, 7), full[3:7])


def _pure_w8a8(X, W):
    """Plain per-token / per-channel symmetric INT8 product (no outlier split),
    vectorised in numpy: the textbook W8A8 linear."""
    x = X.astype(np.float32)
    w = W.astype(np.float32)
    ax = np.abs(x).max(axis=1)
    aw = np.abs(w).max(axis=1)
    with np.errstate(divide="ignore"):
        ix = np.where(ax > 0, np.float32(127) / ax, np.float32(0)).astype(np.float32)
        iw = np.where(aw > 0, np.float32(127) / aw, np.float32(0)).astype(np.float32)
    qx = np.clip(np.rint(x * ix[:, None]), -127, 127).astype(np.int64)
    qw = np.clip(np.rint(w * iw[:, None]), -127, 127).astype(np.int64)
    acc = qx @ qw.T
    sx = (ax / np.float32(127)).astype(np.float64)
    sw = (aw / np.float32(127)).astype(np.float64)
    return acc, acc * sx[:, None] * sw[None, :]


def test_zero_outlier_invariant():
    """No token above T: the layer is exactly the plain W8A8 product."""
    M, K, N = 12, 512, 40
    X = synth.activations(M, K)
    W = synth.weights(N, K)
    idx = synth.outlier_channels(K, 16)
    Xq, s_x, X_out, bitmap, flags = oracle.quantize_act(X, idx, 6.0)
    assert flags[0] == 0 and not X_out.any()
    Wq, s_w, W_out = oracle.prepack_w8(W, idx)
    acc, y = oracle.linear(Xq, s_x, X_out, Wq, s_w, W_out)
    acc_ref, y_ref = _pure_w8a8(X, W)
    np.testing.assert_array_equal(acc, acc_ref)
    np.testing.assert_allclose(y, y_ref, rtol=1e-12, atol=1e-12)


def test_all_outlier_invariant():
    """idx = all K, every token mixed: Xq = 0, acc = 0, Y = X W^T exactly (fp64)."""
    M, K, N = 6, 256, 24
    X = synth.activations(M, K)
    X[:, 0] = 9.0
    W = synth.weights(N, K)
    idx = np.arange(K, dtype=np.int32)
    Xq, s_x, X_out, bitmap, flags = oracle.quantize_act(X, idx, 6.0)
    Wq, s_w, W_out = oracle.prepack_w8(W, idx)
    acc, y = oracle.linear(Xq, s_x, X_out, Wq, s_w, W_out)
    assert flags[0] == M and not acc.any()
    ref = X.astype(np.float64) @ W.astype(np.float64).T
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("k_out,factor", [(0, None), (8, 30.0), (32, None)])
def test_whole_layer_within_quantization_bound(k_out, factor):
    """|Y - X W^T| is bounded by the per-term quantization error of the dense
    part; the outlier part is exact in fp64."""
    M, K, N = 10, 512, 48
    idx = synth.outlier_channels(K, k_out)
    f = factor if factor is not None else synth.channel_factors(k_out)
    X = synth.activations(M, K, idx, f) if k_out else synth.activations(M, K)
    W = synth.weights(N, K)
    Xq, s_x, X_out, bitmap, flags = oracle.quantize_act(X, idx, 6.0)
    Wq, s_w, W_out = oracle.prepack_w8(W, idx)
    _, y = oracle.linear(Xq, s_x, X_out, Wq, s_w, W_out)
    x = X.astype(np.float64)
    w = W.astype(np.float64)
    ref = x @ w.T
    mixed = np.zeros(M, bool)
    in_idx = np.zeros(K, bool)
    in_idx[idx] = True
    for m in range(M):
        mixed[m] = k_out > 0 and np.abs(x[m]).max() > 6.0
    ex = s_x.astype(np.float64) * (0.5 + 1e-4)
    ew = s_w.astype(np.float64) * (0.5 + 1e-4)
    dense = np.where(mixed[:, None] & in_idx[None, :], 0.0, 1.0)
    bound = ((np.abs(x) * dense) @ np.ones((K, N)) * ew[None, :]
             + ex[:, None] * ((dense @ np.abs(w).T))
             + ex[:, None] * ew[None, :] * dense.sum(axis=1, keepdims=True))
    assert (np.abs(y - ref) <= bound + 1e-9).all()
    # and the bound is not vacuous: the quantized layer tracks the exact product
    assert np.abs(y - ref).max() < 0.05 * np.abs(ref).max()


def test_linear_points_match_full():
    (case,) = synth.tiny()
    X, W, idx = case.make()
    Xq, s_x, X_out, _, _ = oracle.quantize_act(X, idx, case.threshold)
    Wq, s_w, W_out = oracle.prepack_w8(W, idx)
    acc, y = oracle.linear(Xq, s_x, X_out, Wq, s_w, W_out)
    ms = np.array([0, 3, 15, 7], np.int32)
    ns = np.array([255, 0, 17, 128], np.int32)
    a2, y2 = oracle.linear_points(Xq, s_x, X_out, Wq, s_w, W_out, ms, ns)
    np.testing.assert_array_equal(a2, acc[ms, ns])
    np.testing.assert_array_equal(y2, y[ms, ns])


def test_round_f16_nearest_even():
    v = np.array([1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, 65504.0, -0.0, 6.0e-8], np.float64)
    got = oracle.round_f16(v)
    np.testing.assert_array_equal(got.astype(np.float64), [1.0, 1.0 + 2.0 ** -9, 65504.0, -0.0,
                                                            np.float16(6.0e-8)])


# ------------------------------------------------- RMS normalisation (next row f1)
def test_rmsnorm_golden_cases(golden_dir):
    g = _load(golden_dir, "rmsnorm_cases.json")
    for c in g["cases"]:
        X = np.asarray([c["x"]], np.float16)
        y = oracle.rmsnorm(X, np.asarray(c["g"], np.float16), c["eps"])
        assert y.view(np.uint16)[0].tolist() == c["y_bits"], c["name"]


def test_rmsnorm_scale_invariance_and_gain():
    # eps = 0: scaling a token by a power of two changes nothing, and scaling the
    # gain by a power of two scales the output exactly (as long as every scaled
    # value stays a normal fp16 number, so the scaling itself is exact)
    X = synth.activations(6, 512)
    g = np.random.default_rng(7).normal(1.0, 0.1, 512).astype(np.float16)
    y = oracle.rmsnorm(X, g, 0.0)
    assert np.abs(X[X != 0]).min() * 0.5 >= 2.0 ** -14 and np.abs(X).max() * 4 < 65504
    for j in (-1, 2):
        Xs = (X.astype(np.float32) * 2.0 ** j).astype(np.float16)
        assert np.array_equal(oracle.rmsnorm(Xs, g, 0.0).view(np.uint16), y.view(np.uint16))
    g2 = (g.astype(np.float32) * 2.0).astype(np.float16)
    assert np.array_equal(oracle.rmsnorm(X, g2, 0.0).astype(np.float32), 2.0 * y.astype(np.float32))


def test_rmsnorm_unit_rms_and_eps():
    # unit gain, eps = 0: every output row has mean square 1 (up to fp16 rounding);
    # eps > 0 shrinks it to ms / (ms + eps)
    X = synth.activations(8, 1024)
    one = np.ones(1024, np.float16)
    ms = (oracle.rmsnorm(X, one, 0.0).astype(np.float64) ** 2).mean(axis=1)
    assert np.all(np.abs(ms - 1.0) < 2e-3)
    x_ms = (X.astype(np.float64) ** 2).mean(axis=1)
    eps = 0.5
    ms_eps = (oracle.rmsnorm(X, one, eps).astype(np.float64) ** 2).mean(axis=1)
    assert np.all(np.abs(ms_eps - x_ms / (x_ms + eps)) < 2e-3)


def test_rmsnorm_rejects_bad_eps():
    X = np.ones((1, 8), np.float16)
    with pytest.raises(oracle.OracleError):
        oracle.rmsnorm(X, np.ones(8, np.float16), -1.0)


# ------------------------------------------------- 4-bit weights, reading B

def _w4b_eff(q, s_g, z_g):
    """Effective weights s * (q - z), fp64, groups expanded along k."""
    s = np.repeat(s_g.astype(np.float64), 128, axis=1)
    z = np.repeat(z_g.astype(np.float64), 128, axis=1)
    return s * (q.astype(np.float64) - z)


def test_w4b_golden_cases(golden_dir):
    g = _load(golden_dir, "w4b_cases.json")
    W = np.zeros((g["rows"], g["K"]), np.float16)
    for c in g["cases"]:
        k0 = 128 * c["group"]
        W[c["row"], k0:k0 + 128] = np.float16(c.get("fill", 0.0))
        for k, v in c["entries"].items():
            W[c["row"], k0 + int(k)] = np.float16(v)
    q, s_g, z_g = oracle.prepack_w4b(W)
    eff = _w4b_eff(q, s_g, z_g)
    for c in g["cases"]:
        r, gi, k0 = c["row"], c["group"], 128 * c["group"]
        assert int(s_g.view(np.uint16)[r, gi]) == c["s_bits"], c["why"]
        assert int(z_g[r, gi]) == c["z"], c["why"]
        for k, qq, e in c["pairs"]:
            assert q[r, k0 + k] == qq, (c["name"], k, c["why"])
            assert eff[r, k0 + k] == e, (c["name"], k, eff[r, k0 + k], e)


def test_w4b_planted_codes_are_recovered():
    """Weights built as s0 * (q - z) with codes 0 and 15 in every group give back
    exactly s0, z and q (s0 varies per group, so a group index mix-up fails)."""
    rng = np.random.default_rng(21)
    N, K = 9, 1024
    ng = K // 128
    choices = np.array([2.0 ** -8, 3 * 2.0 ** -9, 2.0 ** -4, 5 * 2.0 ** -12, 1.0, 0.75])
    s0 = choices[rng.integers(0, len(choices), size=(N, ng))]
    z0 = rng.integers(0, 16, size=(N, ng))
    q0 = rng.integers(0, 16, size=(N, ng, 128))
    q0[:, :, rng.integers(0, 128)] = 0
    q0[:, :, 127 - rng.integers(0, 64)] = 15
    Wexact = s0[:, :, None] * (q0 - z0[:, :, None])
    W = Wexact.reshape(N, K).astype(np.float16)
    assert (W.astype(np.float64) == Wexact.reshape(N, K)).all()  # exact in fp16
    q, s_g, z_g = oracle.prepack_w4b(W)
    np.testing.assert_array_equal(s_g.astype(np.float64), s0)
    np.testing.assert_array_equal(z_g, z0)
    np.testing.assert_array_equal(q, q0.reshape(N, K))
    np.testing.assert_array_equal(_w4b_eff(q, s_g, z_g), W.astype(np.float64))


def test_w4b_round_trip_bound():
    """|s (q - z) - W| <= s/2 plus the fp16 rounding of s (relative 2^-11, times
    at most 15 steps), and the lowest value of a group with a negative entry
    always takes code 0."""
    W = np.concatenate([synth.weights(48, 1024), 3.0 * synth.weights(16, 1024, seed=4) + 0.01])
    W = W.astype(np.float16)
    q, s_g, z_g = oracle.prepack_w4b(W)
    assert q.max() <= 15 and z_g.max() <= 15
    s = np.repeat(s_g.astype(np.float64), 128, axis=1)
    assert (s_g.astype(np.float64) >= 2.0 ** -14).all()  # normal fp16 scales only
    err = np.abs(_w4b_eff(q, s_g, z_g) - W.astype(np.float64))
    eps16 = 2.0 ** -11
    assert (err <= s * (0.5 + 15 * eps16 / (1 - eps16)) + 1e-12).all()
    assert (err / s).max() > 0.45  # the bound is close to tight
    grp = W.reshape(W.shape[0], -1, 128)
    qg = q.reshape(q.shape[0], -1, 128)
    neg = grp.min(axis=2) < 0
    lowest = np.take_along_axis(qg, grp.argmin(axis=2)[:, :, None], axis=2)[:, :, 0]
    assert neg.any() and (lowest[neg] == 0).all()


def test_w4b_one_sided_groups_keep_their_range():
    """The range is widened to hold 0, so an all-positive group gets z = 0 and an
    all-negative one z = 15, and neither loses its extreme value to a clamp."""
    rng = np.random.default_rng(8)
    pos = rng.uniform(0.5, 2.0, 128).astype(np.float16)
    W = np.stack([pos, -pos]).astype(np.float16)
    q, s_g, z_g = oracle.prepack_w4b(W)
    assert list(z_g[:, 0]) == [0, 15]
    assert q[0].max() == 15 and q[1].min() == 0
    err = np.abs(_w4b_eff(q, s_g, z_g) - W.astype(np.float64))
    assert (err <= s_g.astype(np.float64).max() * 0.51).all()


def _w4b_layer_inputs(M, K, N, k_out, seed=0):
    idx = synth.outlier_channels(K, k_out)
    X = synth.activations(M, K, idx, synth.channel_factors(k_out)) if k_out else \
        synth.activations(M, K)
    W = synth.weights(N, K, seed=seed + 1)
    Xq, s_x, X_out, _, _ = oracle.quantize_act(X, idx, synth.THRESHOLD)
    _, _, W_out = oracle.prepack_w8(W, idx)
    q, s_g, z_g = oracle.prepack_w4b(W)
    xo = X_out if X_out.shape[1] else None
    wo = W_out if W_out.shape[1] else None
    return X, W, Xq, s_x, xo, wo, q, s_g, z_g


def test_w4b_layer_brute_force_tiny():
    """Per-group partial sums and the output, in plain Python integers/floats."""
    X, W, Xq, s_x, xo, wo, q, s_g, z_g = _w4b_layer_inputs(3, 256, 4, 64)
    part, y = oracle.linear_w4b(Xq, s_x, xo, q, s_g, z_g, wo)
    for m in range(3):
        for n in range(4):
            acc = 0.0
            for g in range(2):
                p = sum(int(Xq[m, k]) * (int(q[n, k]) - int(z_g[n, g]))
                        for k in range(128 * g, 128 * g + 128))
                assert part[m, n, g] == p
                acc += float(s_g[n, g]) * p
            o = sum(float(xo[m, j]) * float(wo[n, j]) for j in range(xo.shape[1]))
            want = float(s_x[m]) * acc + o
            assert abs(y[m, n] - want) <= 1e-12 * (abs(want) + 1.0)


@pytest.mark.parametrize("M,K,N,k_out", [(7, 1024, 40, 0), (12, 2048, 24, 32), (5, 512, 64, 130)])
def test_w4b_layer_equals_dequantized_product(M, K, N, k_out):
    """The per-group sum equals the product with the dequantized weights
    s (q - z) written out densely (distributivity), and the partial sums equal
    the group slices of an int64 matrix product."""
    X, W, Xq, s_x, xo, wo, q, s_g, z_g = _w4b_layer_inputs(M, K, N, k_out)
    part, y = oracle.linear_w4b(Xq, s_x, xo, q, s_g, z_g, wo)
    wint = q.astype(np.int64) - np.repeat(z_g.astype(np.int64), 128, axis=1)
    for g in range(K // 128):
        sl = slice(128 * g, 128 * g + 128)
        np.testing.assert_array_equal(part[:, :, g], Xq[:, sl].astype(np.int64) @ wint[:, sl].T)
    ref = s_x.astype(np.float64)[:, None] * (Xq.astype(np.float64) @ _w4b_eff(q, s_g, z_g).T)
    if xo is not None:
        ref += xo.astype(np.float64) @ wo.astype(np.float64).T
    np.testing.assert_allclose(y, ref, rtol=1e-11, atol=1e-11)


def test_w4b_layer_tracks_the_exact_product():
    """Against exact X W^T: within the sum of the activation and weight
    quantization errors term by term, and not vacuously."""
    M, K, N, k_out = 9, 1024, 32, 16
    X, W, Xq, s_x, xo, wo, q, s_g, z_g = _w4b_layer_inputs(M, K, N, k_out)
    _, y = oracle.linear_w4b(Xq, s_x, xo, q, s_g, z_g, wo)
    x = X.astype(np.float64)
    w = W.astype(np.float64)
    ref = x @ w.T
    xd = s_x.astype(np.float64)[:, None] * Xq.astype(np.float64)  # dequantized dense part
    xr = x.copy()
    if xo is not None:  # the outlier part of a mixed token is exact
        idx = synth.outlier_channels(K, k_out)
        mixed = np.abs(x).max(axis=1) > synth.THRESHOLD
        xr[np.ix_(mixed, idx)] = 0.0
    weff = _w4b_eff(q, s_g, z_g)
    bound = np.abs(xr - xd) @ np.abs(w).T + np.abs(xd) @ np.abs(weff - w).T
    assert (np.abs(y - ref) <= bound * (1 + 1e-9) + 1e-12).all()
    assert np.abs(y - ref).max() < 0.1 * np.abs(ref).max()


def test_w4b_points_match_full():
    X, W, Xq, s_x, xo, wo, q, s_g, z_g = _w4b_layer_inputs(6, 1024, 40, 16)
    part, y = oracle.linear_w4b(Xq, s_x, xo, q, s_g, z_g, wo)
    ms = np.array([0, 5, 3, 3], np.int32)
    ns = np.array([39, 0, 17, 18], np.int32)
    p2, y2 = oracle.linear_w4b_points(Xq, s_x, xo, q, s_g, z_g, wo, ms, ns)
    np.testing.assert_array_equal(p2, part[ms, ns])
    np.testing.assert_array_equal(y2, y[ms, ns])
