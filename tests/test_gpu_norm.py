"""RMS normalisation absorbed into the activation pass, CUDA path vs the oracle.

The normalised tokens are floating point: the kernel's fp32 result may differ
from the oracle's fp64 result by one fp16 unit in the last place where the exact
value sits next to a rounding boundary.  Every quantization output is an
integer decision, so it is checked bit for bit against the oracle's activation
pass applied to the kernel's own normalised tokens (both sides decide the codes
from the same fp16 values, in fp32).
"""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu

EPS = 1e-5


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    return torch


def _gain(K, seed=11):
    return np.random.default_rng(seed).normal(1.0, 0.1, K).astype(np.float16)


def _ulp_diff(a, b):
    """Distance in fp16 units in the last place (same-sign values; 0 == -0)."""
    ia = a.view(np.uint16).astype(np.int32)
    ib = b.view(np.uint16).astype(np.int32)
    # map sign-magnitude bit patterns onto a monotone integer line
    ia = np.where(ia & 0x8000, -(ia & 0x7FFF), ia)
    ib = np.where(ib & 0x8000, -(ib & 0x7FFF), ib)
    return np.abs(ia - ib)


def _run(torch, X, g, idx, T, with_xn=True):
    import mixed_precision_quantized_mixq_b200 as mq
    Xd = torch.from_numpy(X).cuda()
    gd = torch.from_numpy(g).cuda()
    idxd = torch.from_numpy(np.asarray(idx, np.int32)).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    Xn = torch.full(X.shape, float("nan"), dtype=torch.float16, device="cuda") if with_xn else None
    q = mq.rmsnorm_quantize_act(Xd, gd, EPS, idxd, T, Xn=Xn, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    out = dict(Xq=q.Xq.cpu().numpy(), s_x=q.s_x.cpu().numpy(),
               X_out=(q.X_out.cpu().numpy() if q.X_out is not None
                      else np.zeros((X.shape[0], 0), np.float16)),
               bitmap=q.bitmap.cpu().numpy().view(np.uint32), flags=q.flags.cpu().numpy())
    if with_xn:
        out["Xn"] = Xn.cpu().numpy()
    return out


def _check(g, Xn, idx, T, what):
    Xq, s_x, X_out, bitmap, flags = oracle.quantize_act(Xn, idx, T)
    np.testing.assert_array_equal(g["Xq"], Xq, err_msg=f"{what}: Xq")
    np.testing.assert_array_equal(g["s_x"].view(np.uint32), s_x.view(np.uint32), err_msg=f"{what}: s_x")
    np.testing.assert_array_equal(g["X_out"].view(np.uint16), X_out.view(np.uint16),
                                  err_msg=f"{what}: X_out")
    np.testing.assert_array_equal(g["bitmap"], bitmap, err_msg=f"{what}: bitmap")
    assert list(g["flags"][:2]) == list(flags), (what, g["flags"], flags)
    assert list(g["flags"][2:]) == [0, 0], (what, g["flags"])


def _check_chain(g, X, gain, idx, T, what):
    """The whole chain on the oracle side alone, oracle_rmsnorm then oracle_quantize_act,
    with no value of the kernel as an input: at every token whose scale agrees bit for bit
    with the chain's, every channel whose normalised value agrees has the same code, and a
    token whose normalised outlier channels all agree has the same outlier row.  (A token
    whose amax element lies next to an fp16 rounding boundary may get a scale one step
    apart; those tokens are covered by the check on the kernel's own normalised values.)"""
    ref_n = oracle.rmsnorm(X, gain, EPS)
    Xq, s_x, X_out, _, _ = oracle.quantize_act(ref_n, idx, T)
    same_s = g["s_x"].view(np.uint32) == s_x.view(np.uint32)
    same_x = g["Xn"].view(np.uint16) == ref_n.view(np.uint16)
    mask = same_s[:, None] & same_x
    if X.shape[0] >= 16:
        assert same_s.mean() >= 0.8, f"{what}: {same_s.mean():.3f} of the scales agree"
        assert mask.mean() >= 0.75, f"{what}: {mask.mean():.3f} of the codes compared"
    np.testing.assert_array_equal(g["Xq"][mask], Xq[mask], err_msg=f"{what}: chain Xq")
    if len(idx):
        rows = same_s & same_x[:, np.asarray(idx)].all(axis=1)
        np.testing.assert_array_equal(g["X_out"][rows].view(np.uint16),
                                      X_out[rows].view(np.uint16), err_msg=f"{what}: chain X_out")


@pytest.mark.parametrize("M,K,k_out", [(1, 4096, 64), (16, 4096, 64), (16, 11008, 64),
                                       (64, 4096, 64), (64, 11008, 64), (130, 4096, 128),
                                       (300, 2048, 32), (16, 256, 4), (7, 28672, 128),
                                       (2048, 4096, 256), (33, 1024, 0)])
def test_rmsnorm_quantize_matches_oracle(torch_cuda, M, K, k_out):
    idx = synth.outlier_channels(K, k_out)
    X = synth.activations(M, K, idx, synth.channel_factors(k_out)) if k_out else synth.activations(M, K)
    g = _gain(K)
    T = synth.THRESHOLD
    out = _run(torch_cuda, X, g, idx, T)
    # normalised tokens: within one fp16 ulp of the fp64 oracle, and almost all exact
    ref = oracle.rmsnorm(X, g, EPS)
    d = _ulp_diff(out["Xn"], ref)
    assert d.max() <= 1, f"max ulp difference {d.max()}"
    assert (d > 0).mean() < 0.05, f"{(d > 0).mean():.4f} of the values differ by one ulp"
    # every quantization output bit-exact, decided from the kernel's own normalised tokens
    _check(out, out["Xn"], idx, T, f"M{M} K{K} ko{k_out}")
    # and the oracle's own chain wherever the normalised values agree
    _check_chain(out, X, g, idx, T, f"M{M} K{K} ko{k_out}")
    # the normalised tokens are an optional output: without them the codes are the same
    out2 = _run(torch_cuda, X, g, idx, T, with_xn=False)
    for k in ("Xq", "s_x", "X_out", "bitmap", "flags"):
        np.testing.assert_array_equal(out2[k], out[k], err_msg=f"no-Xn {k}")


def test_rmsnorm_quantize_zero_rows_and_mixed_count(torch_cuda):
    # a zero row normalises to zeros (eps 1e-5 > 0 keeps the denominator positive);
    # scaled outlier channels make the other rows mixed after normalisation
    M, K, k_out = 9, 4096, 64
    idx = synth.outlier_channels(K, k_out)
    X = synth.activations(M, K, idx, synth.channel_factors(k_out))
    X[3] = 0
    out = _run(torch_cuda, X, _gain(K), idx, synth.THRESHOLD)
    assert not out["Xn"][3].any() and not out["Xq"][3].any() and out["s_x"][3] == 0
    _check(out, out["Xn"], idx, synth.THRESHOLD, "zero row")
    assert out["flags"][0] > 0
