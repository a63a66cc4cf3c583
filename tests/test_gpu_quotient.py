"""The quantizers' quotient routine against the IEEE fp32 division.

The INT8 and E4M3 codes are defined on the IEEE fp32 quotient x / delta.  The
pre-pass forms it as RN(q + (x - q delta) y) with y = RN(1 / delta) and q = RN(x y)
(Markstein's theorem, "Computation of elementary functions on the IBM RISC
System/6000 processor", IBM J. Res. Develop. 34, 1990), and divides only where
delta < 2^-60.  Here every finite bf16 and fp16 pattern x is checked against
__fdiv_rn(x, delta) for some six thousand scales delta = RN(amax / 448) and
RN(amax / 127) spread over 2^-60 .. 2^100, including scales right at the threshold,
whole powers of two and amax values that are themselves 16-bit numbers: bit for bit
where the quotient is at least 2^-20, and for every x as the E4M3 code and the
round-half-even integer (smaller quotients, where the quotient or the remainder may be
subnormal, round to the code 0 either way).
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


def _deltas():
    r = np.random.default_rng(20240)
    amax = (np.exp2(r.uniform(-52.0, 100.0, 2500)) * (1.0 + r.random(2500))).astype(np.float32)
    # amax values that are themselves bf16 / fp16 numbers (the usual case: amax of the inputs)
    b16 = (r.integers(0x0080, 0x7F80, 400, dtype=np.uint32) << 16).view(np.float32)
    f16 = r.integers(0x0400, 0x7C00, 400, dtype=np.uint16).view(np.float16).astype(np.float32)
    amax = np.concatenate([amax, b16, f16, np.float32([1.0, 2.0, 448.0, 127.0, 65504.0, 3.0e38])])
    d = np.concatenate([amax / np.float32(448.0), amax / np.float32(127.0)]).astype(np.float32)
    edge = np.float32([2.0 ** -60, np.nextafter(np.float32(2.0 ** -60), np.float32(1.0)), 2.0 ** -59, 1.0, 0.5,
                       1.0 / 3.0, 2.0 ** 20])
    return np.concatenate([d, edge]).astype(np.float32)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_quotient_matches_ieee_division_for_every_16bit_input(dtype):
    deltas = torch.from_numpy(_deltas()).cuda()
    count, first = sage.debug_quotient_check(deltas, dtype)
    assert count == 0, "mismatches %d, first (pattern 0x%04x, delta %r)" % (count, first[0], deltas[first[1]].item())
