"""FP4 (E2M1) quantization with two-level scales on the GPU against the oracle's FP4
Q / K mode, bit for bit: the per-tile fp32 scale, the E4M3 scale of every 16 channels
of a row and every E2M1 code.  (The FP4 QK^T product on the tensor core is the next
step; this checks the quantizer it will consume.)"""
import numpy as np
import pytest
import torch

import oracle
import quantized_attention_fine_b200 as sage
from quantized_attention_fine_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from quantized_attention_fine_b200 import _build
    _build.build()
    sage.load_library()


def _unpack(codes):
    c = codes.cpu().numpy()
    out = np.empty((c.shape[0], c.shape[1] * 2), np.uint8)
    out[:, 0::2] = c & 0xF
    out[:, 1::2] = c >> 4
    return out


@pytest.mark.parametrize("n,d,recipe", [(300, 128, "image_dit"), (200, 64, "llm"), (129, 128, "video_dit")])
def test_fp4_quantizer_bit_exact(n, d, recipe):
    w = wl.custom("fp4", 1, 1, n, n, d, False, recipe=recipe, seed=9900 + n + d)
    q, k, v = (x[0, 0] for x in wl.generate(w))
    pre = oracle.prepass_head(q.double().numpy(), k.double().numpy(), v.double().numpy(), quant=oracle.QK_FP4_PV_FP8)
    n_pad = -(-n // 128) * 128
    for name, x, mean, code, sf, g in (
            ("Q", q, np.repeat(pre["qbar"], 128, axis=0)[:n], pre["q_code"], pre["q_sf"], pre["dq_row"]),
            ("K", k, np.broadcast_to(pre["kbar"], (n, d)), pre["k_code"], pre["k_sf"], pre["dk_key"])):
        xs = (x.float().numpy() - mean.astype(np.float32)).astype(np.float32)   # fp32, as the oracle forms it
        codes_d, sf_d, g_d = sage.debug_quant_fp4(torch.from_numpy(np.ascontiguousarray(xs)).cuda())
        torch.cuda.synchronize()
        got = _unpack(codes_d)
        ref = code[:n_pad].astype(np.uint8)
        assert np.array_equal(g_d.cpu().numpy(), g[::128]), name + ": tile scales"
        assert np.array_equal(sf_d.cpu().numpy(), sf[:n_pad]), name + ": E4M3 block scales"
        if not np.array_equal(got, ref):
            swapped = np.empty_like(got)
            swapped[:, 0::2], swapped[:, 1::2] = got[:, 1::2], got[:, 0::2]
            raise AssertionError("%s: E2M1 codes differ in %d of %d (nibble order swapped matches: %s)"
                                 % (name, int((got != ref).sum()), got.size, np.array_equal(swapped, ref)))
