"""The tensor-core rate loop that gives the tensor-bound GEMMs their measured
peak: it runs to completion without a device error, and its rates are in the
range the B200's dense tensor pipe allows (INT8 about twice the FP16 rate,
both below the nominal dense figures scaled to the highest SM clock)."""
import pytest

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    import mixed_precision_quantized_mixq_b200 as mq
    return torch, mq


def _rate(torch, mq, kind, iters):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    mq.mixq_debug_mma_rate(kind, iters, status)  # warm
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    ops = mq.mixq_debug_mma_rate(kind, iters, status)
    e1.record()
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert ops == sms * iters * 4 * 2 * 128 * 256 * (32 if kind == 0 else 16)
    return ops / (e0.elapsed_time(e1) * 1e-3) / 1e12


def test_int8_and_fp16_rates(env):
    torch, mq = env
    i8 = _rate(torch, mq, 0, 4096)
    f16 = _rate(torch, mq, 1, 4096)
    # dense nominal 4.5 / 2.25 POPS at a boost clock below the 1965 MHz maximum
    assert 1000 < i8 < 5200, i8
    assert 500 < f16 < 2600, f16
    assert 1.6 < i8 / f16 < 2.4, (i8, f16)


def test_rejects_bad_arguments(env):
    torch, mq = env
    for kind, iters in ((2, 16), (0, 0), (1, (1 << 20) + 1)):
        with pytest.raises(mq.MixqError) as e:
            mq.mixq_debug_mma_rate(kind, iters)
        assert e.value.status == 1
