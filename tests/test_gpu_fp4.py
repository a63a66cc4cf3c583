"""FP4 (E2M1) Q / K with two-level scales on the GPU against the oracle's FP4 mode:
the quantizer bit for bit (the per-tile fp32 scale, the E4M3 scale of every 16
channels of a row and every E2M1 code), and one QK^T tile on the block-scaled tensor
core (tcgen05.mma kind::mxf4nvf4 with the scales in tensor memory) against the
oracle's dequantized scores, up to the order of the fp32 sum."""
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


def _pack(codes):
    c = np.asarray(codes, np.uint8)
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


@pytest.mark.parametrize("d", [64, 128])
def test_fp4_qk_tile_on_the_tensor_core(d):
    """S[i][j] = sum_c sf_q e2m1_q * sf_k e2m1_k from the oracle's codes and scales (its
    q_hat, k_hat), accumulated exactly in fp64, against the tensor core's fp32 sum: each
    16-channel block's partial is exact in fp32, so only the order of the block sums
    rounds (relative 2^-22 of the sum of magnitudes, d / 16 terms)."""
    w = wl.custom("fp4qk", 1, 1, 128, 128, d, False, recipe="image_dit", seed=7700 + d)
    q, k, v = (x[0, 0] for x in wl.generate(w))
    pre = oracle.prepass_head(q.double().numpy(), k.double().numpy(), v.double().numpy(), quant=oracle.QK_FP4_PV_FP8)
    q4 = torch.from_numpy(_pack(pre["q_code"][:128])).cuda()
    k4 = torch.from_numpy(_pack(pre["k_code"][:128])).cuda()
    sfq = torch.from_numpy(np.ascontiguousarray(pre["q_sf"][:128])).cuda()
    sfk = torch.from_numpy(np.ascontiguousarray(pre["k_sf"][:128])).cuda()
    s = sage.debug_qk_tile_fp4(q4, k4, sfq, sfk).cpu().double().numpy()
    ref = pre["q_hat"][:128] @ pre["k_hat"][:128].T
    bound = np.abs(pre["q_hat"][:128]) @ np.abs(pre["k_hat"][:128]).T * (d // 16) * 2.0 ** -23 + 1e-30
    err = np.abs(s - ref)
    assert np.all(err <= bound), "max err %.3g (bound %.3g)" % (err.max(), bound[np.argmax(err - bound)])
    # a transposed or mis-scaled tile would not be this close
    assert np.corrcoef(s.ravel(), ref.ravel())[0, 1] > 0.999999
