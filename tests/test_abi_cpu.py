"""The C ABI library on a machine without a GPU: it loads, exports every symbol
include/mixq.h declares, and does its host-side work (argument checks, size
queries, launch planning) without touching a device."""
import ctypes

import numpy as np
import os
import re

import pytest

import mixed_precision_quantized_mixq_b200 as mq
from mixed_precision_quantized_mixq_b200 import build as mqbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    mqbuild.build()
    return mq.lib()


def _declared():
    with open(os.path.join(ROOT, "include", "mixq.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"\b(mixq_[a-z0-9_]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = _declared()
    assert len(names) >= 11
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(mq._SIGNATURES), "binding signatures out of sync with the header"


def test_version(lib):
    assert lib.mixq_version() == 100


def test_no_gemm_workspace(lib):
    for M, N, K in ((1, 128, 128), (16, 11008, 4096), (8192, 28672, 8192)):
        assert lib.mixq_gemm_workspace_size(M, N, K) == 0


def test_prepack_size(lib):
    assert mq.mixq_prepack_size(mq.MIXQ_W8, 256, 512, 4) == (256 * 512, 0, 2 * 256 * 64)
    assert mq.mixq_prepack_size(mq.MIXQ_W4G128, 256, 512, 65) == (256 * 256, 4 * 256 * 4,
                                                                  2 * 256 * 128)
    assert mq.mixq_prepack_size(mq.MIXQ_W8, 128, 128, 0)[2] == 0


@pytest.mark.parametrize("N,K,K_out", [(100, 128, 0), (128, 100, 0), (0, 128, 0), (128, 128, 129),
                                       (128, 128, -1)])
def test_shape_rules(lib, N, K, K_out):
    with pytest.raises(mq.MixqError) as e:
        mq.mixq_prepack_size(mq.MIXQ_W8, N, K, K_out)
    assert e.value.status == 2
    assert "must" in lib.mixq_last_error().decode()


def test_bad_mode(lib):
    with pytest.raises(mq.MixqError) as e:
        mq.mixq_prepack_size(7, 128, 128, 0)
    assert e.value.status == 1


def test_host_checks_come_before_device_checks(lib):
    # misaligned pointers are reported without any device access
    rc = lib.mixq_gemm_w8a8o16(4, 256, 256, 0, 0x1001, 0x2000, None, 0x3000, 0x4000, None, None,
                               0x5000, 256, None, None)
    assert rc == 3
    rc = lib.mixq_gemm_w8a8o16(4, 256, 256, 0, None, 0x2000, None, 0x3000, 0x4000, None, None,
                               0x5000, 256, None, None)
    assert rc == 1
    rc = lib.mixq_gemm_w8a8o16(4, 256, 256, 0, 0x1000, 0x2000, None, 0x3000, 0x4000, None, None,
                               0x5000, 250, None, None)
    assert rc == 1
    rc = lib.mixq_quantize_act(0x1000, 4, 256, 256, None, 0, ctypes.c_float(-1.0), 0x2000, 0x3000,
                               None, 0x4000, 0x5000, None, None)
    assert rc == 1


def test_rmsnorm_quantize_host_checks(lib):
    f = ctypes.c_float
    # null gain, negative / NaN eps, short Xn stride, misaligned gain: all host errors
    args = dict(X=0x1000, M=4, K=256, ldx=256, gamma=0x6000, eps=f(1e-5), Xn=None, ldxn=0,
                idx=None, K_out=0, T=f(6.0), Xq=0x2000, s_x=0x3000, X_out=None, bitmap=0x4000,
                flags=0x5000, status=None, stream=None)

    def call(**kw):
        a = dict(args, **kw)
        return lib.mixq_rmsnorm_quantize_act(*a.values())

    assert call(gamma=None) == 1
    assert call(eps=f(-1.0)) == 1
    assert call(eps=f(float("nan"))) == 1
    assert call(Xn=0x7000, ldxn=128) == 1
    assert call(gamma=0x6008) == 3


def _merge(lib, bitmap, idx, K):
    bitmap = np.ascontiguousarray(bitmap, np.uint32)
    idx = np.ascontiguousarray(idx, np.int32)
    out = np.full(K, -1, np.int32)
    n = ctypes.c_int(-1)
    rc = lib.mixq_merge_outliers(bitmap.ctypes.data, K, idx.ctypes.data if idx.size else None,
                                 idx.size, out.ctypes.data, ctypes.byref(n))
    return rc, out[:max(n.value, 0)]


def test_merge_outliers_is_the_sorted_union(lib):
    # host-only call: the outlier set grows by the channels detected outside it
    rng = np.random.default_rng(3)
    for K in (32, 256, 4096):
        for _ in range(20):
            idx = np.sort(rng.choice(K, rng.integers(0, K // 4 + 1), replace=False)).astype(np.int32)
            det = rng.choice(K, rng.integers(0, K // 8 + 1), replace=False)
            bitmap = np.zeros(K // 32, np.uint32)
            for c in det:
                bitmap[c // 32] |= np.uint32(1) << np.uint32(c % 32)
            rc, got = _merge(lib, bitmap, idx, K)
            assert rc == 0
            np.testing.assert_array_equal(got, np.union1d(idx, det).astype(np.int32))
    # all channels detected -> every channel; nothing detected -> idx unchanged
    rc, got = _merge(lib, np.full(8, 0xFFFFFFFF, np.uint32), np.array([5, 9], np.int32), 256)
    assert rc == 0 and np.array_equal(got, np.arange(256))
    rc, got = _merge(lib, np.zeros(8, np.uint32), np.array([5, 9], np.int32), 256)
    assert rc == 0 and np.array_equal(got, [5, 9])


def test_merge_outliers_rejects_bad_input(lib):
    z = np.zeros(8, np.uint32)
    assert _merge(lib, z, np.array([9, 5], np.int32), 256)[0] == 1      # unsorted
    assert _merge(lib, z, np.array([5, 5], np.int32), 256)[0] == 1      # duplicate
    assert _merge(lib, z, np.array([-1], np.int32), 256)[0] == 1        # out of range
    assert _merge(lib, z, np.array([300], np.int32), 256)[0] == 1       # out of range
    assert _merge(lib, np.zeros(1, np.uint32), np.array([], np.int32), 33)[0] == 1  # K % 32


def test_no_device_reported(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    rc = lib.mixq_gemm_w8a8o16(4, 256, 256, 0, 0x1000, 0x2000, None, 0x3000, 0x4000, None, None,
                               0x5000, 256, None, None)
    assert rc == 6
    assert "device" in lib.mixq_last_error().decode()


@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (16, 11008, 4096), (64, 4096, 11008),
                                   (512, 4096, 4096), (2048, 11008, 4096), (8192, 11008, 4096),
                                   (512, 28672, 8192), (512, 8192, 28672)])
def test_gemm_plan(lib, M, N, K):
    bn, split, ctas = mq.mixq_gemm_plan(mq.MIXQ_W8, M, N, K, 148)
    assert bn in (32, 64, 128, 256) and 1 <= split <= 8 and split <= K // 128
    assert bn >= 128 or M <= 64
    tiles256 = -(-M // 256) * -(-N // 256)
    if M >= 256:
        # persistent CTA-pair kernel: 256 x 256 tiles, one pair per two SMs
        assert bn == 256 and split == 1 and ctas == 2 * min(tiles256, 74)
        return
    assert ctas == -(-M // 128) * -(-N // bn) * split
    if M <= 64:
        # decode: narrow tiles and/or a K split across a cluster so that most
        # SMs stream weights
        assert ctas >= 64
    if M >= 2048:
        assert split == 1


@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (16, 11008, 4096), (64, 4096, 11008),
                                   (100, 4096, 4096), (200, 4096, 4096), (512, 4096, 4096),
                                   (2048, 11008, 4096), (512, 28672, 8192), (512, 8192, 28672)])
def test_gemm_plan_w4(lib, M, N, K):
    bn, split, ctas = mq.mixq_gemm_plan(mq.MIXQ_W4G128, M, N, K, 148)
    assert 1 <= split <= 8 and split <= K // 128
    if M <= 64:
        # tensor-memory-operand kernel: 128 weight rows x all tokens per tile
        assert bn == 128 and ctas == (N // 128) * split
        assert 64 <= ctas <= 2 * 148
    elif M >= 2048:
        # persistent CTA-pair kernel: 256 weight rows x 256 tokens per pair of SMs
        tiles = -(-M // 256) * -(-N // 256)
        assert bn == 256 and split == 1 and ctas == 2 * min(tiles, 74)
    elif M > 1024 or (M >= 256 and -(-M // 128) * (N // 128) * 5 < 148 * 4):
        # tensor-memory-operand kernel, one CTA per SM with 256-token tiles
        assert bn == 128 and split == 1 and ctas == -(-M // 256) * (N // 128)
    else:
        # tensor-memory-operand kernel, 128-token tiles
        assert bn == 128 and ctas == -(-M // 128) * (N // 128) * split


# ------------------------------------ 4-bit weights with an fp16 group scale

def test_prepack_size_f16s(lib):
    # same packed code and group-pair sizes as the progressive 4-bit format
    for N, K, ko in ((256, 512, 65), (4096, 11008, 64), (128, 128, 0)):
        assert mq.mixq_prepack_size(mq.MIXQ_W4G128_F16S, N, K, ko) == \
            mq.mixq_prepack_size(mq.MIXQ_W4G128, N, K, ko)


@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (16, 11008, 4096), (16, 4096, 11008),
                                   (8, 256, 1024), (17, 11008, 4096),
                                   (40, 4096, 4096), (64, 256, 1024), (100, 4096, 4096),
                                   (2048, 11008, 4096), (512, 8192, 28672)])
def test_gemm_plan_f16s(lib, M, N, K):
    """M <= 16: the two-CTA-per-SM variant (16 tokens per tile), K split as the
    other decode kernels: the smallest split reaching 0.8 CTA per SM with <= 11
    K blocks per CTA, never past two CTAs per SM.  Otherwise one CTA per SM with
    all tokens (M <= 64) or 64 tokens per tile; a K split only while the tiles
    leave SMs idle, never past one wave, at most 8 and at most K/128; the
    smallest split reaching 0.8 CTA per SM with <= 11 K blocks per CTA."""
    sms, KB = 148, K // 128
    bn, split, ctas = mq.mixq_gemm_plan(mq.MIXQ_W4G128_F16S, M, N, K, sms)
    assert 1 <= split <= min(8, KB)
    if M <= 16:
        tiles = N // 128
        assert bn == 128 and ctas == tiles * split and ctas <= 2 * sms
        for s in range(1, split):
            assert not (tiles * s * 5 >= sms * 4 and -(-KB // s) <= 11)
        assert (ctas * 5 >= sms * 4 and -(-KB // split) <= 11) or split == min(8, KB) or \
            tiles * (split + 1) > 2 * sms
        return
    tiles = -(-M // 64) * (N // 128)
    assert bn == 128 and ctas == tiles * split
    if split > 1:
        assert ctas <= sms
        # no smaller split already met the occupancy and depth goal
        for s in range(1, split):
            assert not (tiles * s * 5 >= sms * 4 and -(-KB // s) <= 11)
        # and the chosen one meets it, or the next one would overflow the wave
        assert (ctas * 5 >= sms * 4 and -(-KB // split) <= 11) or split == min(8, KB) or \
            tiles * (split + 1) > sms
    else:
        assert tiles * 5 >= sms * 4 or tiles * 2 > sms or KB == 1


def test_gemm_plan_f16s_examples(lib):
    # decode N = 11008: 86 tiles x 3 = 258 CTAs (two per SM), 10-11 K blocks each
    assert mq.mixq_gemm_plan(mq.MIXQ_W4G128_F16S, 16, 11008, 4096, 148) == (128, 3, 258)
    # decode N = 4096, K = 4096: 32 tiles x 4 = 128 CTAs, 8 K blocks each
    assert mq.mixq_gemm_plan(mq.MIXQ_W4G128_F16S, 16, 4096, 4096, 148) == (128, 4, 128)
    # decode K = 11008: 32 tiles x 8 = 256 CTAs, 10-11 K blocks each
    assert mq.mixq_gemm_plan(mq.MIXQ_W4G128_F16S, 1, 4096, 11008, 148) == (128, 8, 256)
    # 17..64 tokens: one CTA per SM; N = 11008 needs a second wave for split 2
    assert mq.mixq_gemm_plan(mq.MIXQ_W4G128_F16S, 64, 11008, 4096, 148) == (128, 1, 86)
    # small layer: 4 tiles, split 8 (K = 1024: one K block per CTA)
    assert mq.mixq_gemm_plan(mq.MIXQ_W4G128_F16S, 100, 256, 1024, 148) == (128, 8, 32)


def test_f16s_host_checks(lib):
    # the scale-free format takes no s_w: a null s_w passes the host checks (the
    # call then stops at the missing device), a null Xq or a bad ldy does not
    g = lib.mixq_gemm_w4a8o16_f16s
    assert g(4, 256, 256, 0, None, 0x2000, None, 0x3000, 0x4000, None, None, 0x5000, 256, None,
             None) == 1
    assert g(4, 256, 256, 0, 0x1000, 0x2000, None, 0x3000, None, None, None, 0x5000, 256, None,
             None) == 1  # grp missing
    assert g(4, 256, 256, 0, 0x1000, 0x2000, None, 0x3000, 0x4000, None, None, 0x5000, 250, None,
             None) == 1
    assert g(4, 256, 256, 0, 0x1000, 0x2000, None, 0x3008, 0x4000, None, None, 0x5000, 256, None,
             None) == 3
    assert g(4, 256, 200, 0, 0x1000, 0x2000, None, 0x3000, 0x4000, None, None, 0x5000, 256, None,
             None) == 2
    # prepack: s_w may be null for this format only
    p = lib.mixq_prepack_weights
    assert p(mq.MIXQ_W4G128, 0x1000, 256, 256, None, 0, 0x2000, None, 0x3000, None, None,
             None) == 1
    assert p(mq.MIXQ_W4G128_F16S, 0x1000, 256, 256, None, 0, 0x2000, None, None, None, None,
             None) == 1  # grp missing
    import torch
    if not torch.cuda.is_available():
        assert g(4, 256, 256, 0, 0x1000, 0x2000, None, 0x3000, 0x4000, None, None, 0x5000, 256,
                 None, None) == 6
        assert p(mq.MIXQ_W4G128_F16S, 0x1000, 256, 256, None, 0, 0x2000, None, 0x3000, None,
                 None, None) == 6


def test_mma_rate_argument_checks(lib):
    # host-side checks come before any device access
    import ctypes as c
    ops = c.c_double()
    assert lib.mixq_debug_mma_rate(2, 16, c.byref(ops), None, None) == 1
    assert lib.mixq_debug_mma_rate(0, 0, c.byref(ops), None, None) == 1
    assert lib.mixq_debug_mma_rate(0, 16, None, None, None) == 1
