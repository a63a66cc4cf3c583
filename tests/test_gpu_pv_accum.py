"""The FP16-accumulator form of the FP8 PV product (the instruction SageAttention2++
moves PV to, with the range narrowing Pr * Vr <= 2047/2) on the B200 tensor core,
and the throughput of each tcgen05.mma form the forward uses.

The forward itself accumulates PV in FP32 (test_fp8_pv_accumulates_in_full_fp32);
these tests measure what the FP16 accumulator would change.
"""
import numpy as np
import pytest
import torch

import quantized_attention_fine_b200 as sage

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from quantized_attention_fine_b200 import _build
    _build.build()
    sage.load_library()


def _e4m3(x):
    return torch.as_tensor(x, dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8)


def _run(p, v):
    raw = sage.debug_pv_accumulate_f16acc(_e4m3(p).cuda(), _e4m3(v).cuda()).cpu().numpy().astype(np.uint32)
    lo, hi = raw & 0xFFFF, raw >> 16
    return lo, hi


def _f16(bits):
    return bits.astype(np.uint16).view(np.float16).astype(np.float64)


def _decode(lo, hi):
    """FP16 values of the accumulator words: the half that holds them (the other is 0)."""
    if not hi.any():
        return _f16(lo)
    assert not lo.any(), "neither half of the accumulator words is empty"
    return _f16(hi)


@pytest.mark.parametrize("d", [64, 128])
def test_fp16_accumulator_exact_sums(d):
    """Sums that FP16 holds exactly (multiples of 0.5 up to 128) come out exact."""
    T = 2
    p = torch.ones((T, 128, 128))
    v = torch.full((T, d, 128), 0.5)
    v[:, 1::2] = -0.5
    o = _decode(*_run(p, v))
    expect = np.where(np.arange(d) % 2 == 0, 64.0 * T, -64.0 * T)
    assert np.array_equal(o, np.broadcast_to(expect, o.shape))


def test_fp16_accumulator_loses_low_bits():
    """448 plus 127 products of 2^-8: exact in FP32 (the forward's accumulator), not in
    FP16, whose spacing at 448 is 0.25."""
    d = 64
    p = torch.zeros((1, 128, 128))
    v = torch.zeros((1, d, 128))
    p[:, :, 0] = 448.0
    v[:, :, 0] = 1.0
    p[:, :, 1:] = 2.0 ** -4
    v[:, :, 1:] = 2.0 ** -4
    o = _decode(*_run(p, v))
    exact = 448.0 + 127 * 2.0 ** -8
    assert np.all(o != exact)
    assert np.all(np.abs(o - exact) <= 4 * 0.25)   # at most one FP16 rounding per 32-key MMA


def test_fp16_accumulator_needs_the_range_bound():
    """With SageAttention2++'s ranges Pr = 224, Vr = 4.5 (Pr Vr = 1008 <= 2047/2), 64
    products stay finite (64 * 1008 = 64512 <= 65504): two 32-key MMAs may share an
    FP16 accumulator.  128 of them overflow: a whole 128-key tile may not."""
    d = 64
    v = torch.full((1, d, 128), 4.5)
    p64 = torch.zeros((1, 128, 128))
    p64[:, :, :64] = 224.0
    o = _decode(*_run(p64, v))
    assert np.all(o == 64512.0)
    p128 = torch.full((1, 128, 128), 224.0)
    o = _decode(*_run(p128, v))
    assert np.all(~np.isfinite(o) | (o >= 65504.0))


def test_mma_rates():
    """Throughput of each tcgen05.mma form (M = 128, N = 256), one CTA per SM."""
    rates = {k: sage.debug_mma_rate(k) for k in sage.MMA_KINDS}
    print("tcgen05.mma dense rates (TFLOP/s, TOPS for s8):", {k: round(r, 1) for k, r in rates.items()})
    for k, r in rates.items():
        assert 100.0 < r < 20000.0, (k, r)
