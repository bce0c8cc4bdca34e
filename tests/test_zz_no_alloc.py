"""mixq_quantize_act_static, the activation pass for callers that cannot
allocate device memory (a runtime plugin handed fixed buffers, code whose
memory belongs to another allocator, a hot path where cudaMalloc's possible
device synchronisation is not acceptable): its completion ticket lives in a
256-byte array inside the library instead of two extra caller flag words.

Called through the C ABI, two calls in a row on different inputs, each
compared bit for bit with mixq_quantize_act on the same input (codes, scales,
outlier columns, detection bitmap and both flag words are exact outputs, so
the tolerance is zero).  The second call only comes out right if the first
left the shared scratch in a state the next call can use.  Shapes cover the
single-cluster pass (no ticket) and the multi-CTA pass (ticket).
"""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    import mixed_precision_quantized_mixq_b200 as mq
    mq.lib()
    return torch, mq


def _inputs(M, K, k_out, seed):
    """Seeded activations with the outlier channels scaled, plus three channels
    outside the list scaled too (detections the list does not hold)."""
    idx = synth.outlier_channels(K, k_out)
    X = synth.activations(M, K, idx, synth.channel_factors(k_out), seed=seed)
    rng = np.random.default_rng(seed + 100)
    extra = rng.choice(np.setdiff1d(np.arange(K), idx), size=3, replace=False)
    X[:, extra] = (X[:, extra].astype(np.float32) * 30).astype(np.float16)
    return X, idx


def _outputs(torch, M, K, k_out, flag_words):
    kp = (k_out + 63) // 64 * 64
    return dict(Xq=torch.full((M, K), 99, dtype=torch.int8, device="cuda"),
                s_x=torch.full((M,), -1.0, dtype=torch.float32, device="cuda"),
                X_out=torch.full((M, kp), 7.0, dtype=torch.float16, device="cuda") if kp else None,
                bitmap=torch.full((K // 32,), -1, dtype=torch.int32, device="cuda"),
                flags=torch.full((flag_words,), 12345, dtype=torch.int32, device="cuda"))


def _host(o):
    return {k: (None if v is None else v.cpu().numpy()) for k, v in o.items()}


@pytest.mark.parametrize("M,K,k_out", [(16, 4096, 64), (300, 4096, 64), (40, 11008, 64),
                                       (100, 16384, 32), (8, 2048, 0)])
def test_static_scratch_matches_quantize_act(env, M, K, k_out):
    torch, mq = env
    T = synth.THRESHOLD
    for call, seed in enumerate((5, 6)):
        X, idx = _inputs(M, K, k_out, seed)
        Xd = torch.from_numpy(X).cuda()
        idxd = torch.from_numpy(idx).cuda() if k_out else None
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        ref = _outputs(torch, M, K, k_out, 4)
        mq.mixq_quantize_act(Xd, idxd, T, ref["Xq"], ref["s_x"], ref["X_out"], ref["bitmap"],
                             ref["flags"], status)
        new = _outputs(torch, M, K, k_out, 2)
        mq.mixq_quantize_act_static(Xd, idxd, T, new["Xq"], new["s_x"], new["X_out"],
                                    new["bitmap"], new["flags"], status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        r, n = _host(ref), _host(new)
        what = f"call {call + 1}, M{M} K{K} ko{k_out}"
        np.testing.assert_array_equal(n["Xq"], r["Xq"], err_msg=what)
        np.testing.assert_array_equal(n["s_x"].view(np.uint32), r["s_x"].view(np.uint32),
                                      err_msg=what)
        if k_out:
            np.testing.assert_array_equal(n["X_out"].view(np.uint16), r["X_out"].view(np.uint16),
                                          err_msg=what)
        np.testing.assert_array_equal(n["bitmap"], r["bitmap"], err_msg=what)
        np.testing.assert_array_equal(n["flags"], r["flags"][:2], err_msg=what)
        # the three planted channels outside the list are detected
        assert n["flags"][1] >= (3 if k_out else 0), what
