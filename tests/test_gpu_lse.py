"""Row log-sum-exp (LSE) output of the attention step, through the C ABI.

The LSE is of the logits the method computes (quantized scores plus dS), referred back
to the unsmoothed logits by the per-row shift (q_i - qbar_t) . kbar that the pre-pass
stores.  GPU and oracle make the same integer decisions, so the two agree to fp32
rounding of the exponent sums and of the shift.
"""
import numpy as np
import pytest
import torch

import oracle
import quantized_attention_fine_b200 as sage
from quantized_attention_fine_b200 import workloads as wl

from helpers import GRAN_OF, O_COS_FULL, cos, head_slices, to_np64

pytestmark = pytest.mark.gpu

LSE_MAX_ABS = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from quantized_attention_fine_b200 import _build
    _build.build()
    sage.load_library()


def _assert_lse_close(got, ref, what):
    fin = np.isfinite(ref)
    assert np.array_equal(np.isfinite(got), fin), "%s: finite pattern differs" % what
    assert np.all(got[~fin] == -np.inf), "%s: rows without keys must be -inf" % what
    if fin.any():
        err = np.max(np.abs(got[fin] - ref[fin]))
        assert err <= LSE_MAX_ABS, "%s: max |LSE_gpu - LSE_oracle| = %.3e" % (what, err)


LSE_CASES = [
    # name, B, H, H_kv, nq, nk, d, causal, layout, recipe, kwargs
    ("ragged_causal_d128", 1, 2, 2, 600, 600, 128, True, "HND", "llm", {}),
    ("q_longer_causal_d64", 1, 2, 2, 520, 300, 64, True, "NHD", "image_dit", {}),
    ("kv_longer_d64", 2, 1, 1, 300, 520, 64, False, "HND", "video_dit", {}),
    ("gqa_g4_causal", 1, 8, 2, 333, 333, 128, True, "HND", "sweep", {}),
    ("smoothing_off", 1, 2, 2, 384, 384, 128, False, "HND", "image_dit", dict(smooth_q=False, smooth_k=False)),
    ("smooth_k_only_per_block", 1, 2, 2, 300, 300, 64, True, "NHD", "llm",
     dict(smooth_q=False, granularity="per_block")),
]


@pytest.mark.parametrize("name,B,H,Hk,nq,nk,d,causal,layout,recipe,kw", LSE_CASES, ids=[c[0] for c in LSE_CASES])
def test_lse_matches_oracle(name, B, H, Hk, nq, nk, d, causal, layout, recipe, kw):
    w = wl.custom(name, B, H, nq, nk, d, causal, recipe=recipe, H_kv=Hk, seed=8100 + nq + nk + d + H)
    q, k, v = wl.generate(w)
    if layout == "NHD":
        q, k, v = wl.to_nhd(q), wl.to_nhd(k), wl.to_nhd(v)
    o, lse = sage.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, layout=layout, return_lse=True, **kw)
    lse = lse.cpu().double().numpy()
    assert lse.shape == (B, H, nq)
    gran = kw.get("granularity", "per_threadgroup")
    g_q, g_k = GRAN_OF[gran]
    group = H // Hk
    for b in range(B):
        for h in range(H):
            qh = head_slices(q, q, q, b, h, layout)[0]
            kh, vh = head_slices(k, k, v, b, h // group, layout)[1:]
            pre = oracle.prepass_head(to_np64(qh), to_np64(kh), to_np64(vh), g_q=g_q, g_k=g_k,
                                      smooth_q=kw.get("smooth_q", True), smooth_k=kw.get("smooth_k", True))
            _assert_lse_close(lse[b, h], oracle.lse_head(pre, causal=causal), "%s b%d h%d" % (name, b, h))


def test_row_shift_matches_fp64():
    """The stored shift (q_i - qbar_t) . kbar against the same product in fp64 from the
    workspace's own qbar and kbar (fp32 rounding of the terms and the sum only)."""
    B, H, n, d = 1, 2, 300, 128
    w = wl.custom("shift", B, H, n, n, d, False, recipe="image_dit", seed=8200)
    q, k, v = wl.generate(w)
    ws = sage.quant_qk(q.cuda(), k.cuda())
    torch.cuda.synchronize()
    shift = ws.view("qs_kbar").cpu().double().numpy()
    qbar = ws.view("qbar").cpu().double().numpy()
    kbar = ws.view("kbar").cpu().double().numpy()
    for h in range(H):
        qs = to_np64(q[0, h]) - np.repeat(qbar[h], 128, axis=0)[:n]
        ref = qs @ kbar[h]
        scale = np.abs(qs) @ np.abs(kbar[h]) + 1e-30
        assert np.max(np.abs(shift[h, :n] - ref) / scale) < 1e-5


def test_lse_merges_partial_outputs_over_key_ranges():
    """Two calls over the two halves of the keys (each with its own K mean, so their
    smoothed logits are shifted differently) merge by their LSEs into the attention over
    all keys: softmax weights exp(LSE_1) and exp(LSE_2)."""
    B, H, nq, nk, d = 1, 2, 256, 640, 128
    w = wl.custom("merge", B, H, nq, nk, d, False, recipe="llm", seed=8300)
    q, k, v = (x.cuda() for x in wl.generate(w))
    cut = 384
    o1, l1 = sage.attn_fwd(q, k[:, :, :cut].contiguous(), v[:, :, :cut].contiguous(), return_lse=True)
    o1, l1 = o1.double(), l1.double().clone()
    o2, l2 = sage.attn_fwd(q, k[:, :, cut:].contiguous(), v[:, :, cut:].contiguous(), return_lse=True)
    o2, l2 = o2.double(), l2.double().clone()
    lse = torch.logaddexp(l1, l2)
    o = (torch.exp(l1 - lse)[..., None] * o1 + torch.exp(l2 - lse)[..., None] * o2).cpu().numpy()
    o_full, l_full = sage.attn_fwd(q, k, v, return_lse=True)
    qn, kn, vn = (to_np64(x.cpu()) for x in (q, k, v))
    ref = oracle.reference_attention(qn, kn, vn)
    assert cos(o, ref) >= O_COS_FULL
    assert cos(o_full.double().cpu().numpy(), ref) >= O_COS_FULL
    # the merged LSE and the one-call LSE are both close to the exact log-sum-exp
    x = torch.from_numpy(qn @ kn.transpose(0, 1, 3, 2)) / np.sqrt(d)
    exact = torch.logsumexp(x, dim=-1).numpy()
    assert np.max(np.abs(lse.cpu().numpy() - exact)) < 0.05
    assert np.max(np.abs(l_full.double().cpu().numpy() - exact)) < 0.05
