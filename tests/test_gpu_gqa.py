"""Grouped-query attention on the GPU, through the C ABI (the `_gqa` entry points).

H query heads share H_kv key/value heads; query head h reads key/value head
h // (H // H_kv).  The pre-pass is checked bit-exact per key/value head (K codes,
delta_K, K mean, V codes, delta_V) and per query head (Q codes, delta_Q, Q block
means, dS over the key/value head's K); the attention output of every query head
against the oracle run on that head and its key/value head.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import quantized_attention_fine_b200 as sage
from quantized_attention_fine_b200 import workloads as wl

from helpers import O_COS_FULL, GRAN_OF, assert_close_to_oracle, cos, natural_key_order, oracle_head, to_np64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from quantized_attention_fine_b200 import _build
    _build.build()
    sage.load_library()


def _inputs(B, H, H_kv, nq, nk, d, causal, layout="HND", recipe="llm", dtype=torch.bfloat16, seed=7000):
    w = wl.custom("gqa", B, H, nq, nk, d, causal, dtype=dtype, recipe=recipe, H_kv=H_kv,
                  seed=seed + 31 * H + 7 * H_kv + nq + 3 * nk + d)
    q, k, v = wl.generate(w)
    if layout == "NHD":
        q, k, v = wl.to_nhd(q), wl.to_nhd(k), wl.to_nhd(v)
    return q, k, v


def _head(x, b, h, layout):
    return x[b, h] if layout == "HND" else x[b, :, h]


PREPASS_CASES = [
    # B, H, H_kv, nq, nk, d, layout, granularity
    (2, 4, 2, 300, 520, 128, "HND", "per_threadgroup"),
    (1, 6, 1, 200, 333, 64, "NHD", "per_threadgroup"),
    (1, 8, 2, 130, 260, 128, "NHD", "per_warp"),
]


@pytest.mark.parametrize("B,H,Hk,nq,nk,d,layout,gran", PREPASS_CASES)
def test_gqa_prepass_bit_exact(B, H, Hk, nq, nk, d, layout, gran):
    q, k, v = _inputs(B, H, Hk, nq, nk, d, False, layout=layout)
    mode = sage.QuantMode.make(gran)
    ws = sage.quant_qk(q.cuda(), k.cuda(), layout=layout, mode=mode)
    assert ws.H_kv == Hk
    sage.quant_v(v.cuda(), n_q=nq, layout=layout, mode=mode, workspace=ws)
    torch.cuda.synchronize()
    views = {n: ws.view(n).cpu() for n in sage.WS_VIEWS}
    assert views["k8"].shape[0] == B * Hk and views["q8"].shape[0] == B * H
    g_q, g_k = GRAN_OF[gran]
    group = H // Hk
    for b in range(B):
        for h in range(H):
            bh, bk = b * H + h, b * Hk + h // group
            qh, kh, vh = _head(q, b, h, layout), _head(k, b, h // group, layout), _head(v, b, h // group, layout)
            pre = oracle.prepass_head(to_np64(qh), to_np64(kh), to_np64(vh), g_q=g_q, g_k=g_k)
            assert np.array_equal(views["qbar"][bh].numpy(), pre["qbar"]), "qbar"
            assert np.array_equal(views["dq"][bh].numpy(), pre["dq_row"]), "delta_Q"
            assert np.array_equal(views["q8"][bh].numpy(), pre["q_code"]), "Q codes"
            if h % group == 0:  # the key/value head's arrays, once per key/value head
                assert np.array_equal(views["kbar"][bk].numpy(), pre["kbar"]), "kbar"
                assert np.array_equal(views["dk"][bk].numpy(), pre["dk_key"][::16]), "delta_K"
                assert np.array_equal(views["dv"][bk].numpy(), pre["dv"]), "delta_V"
                assert np.array_equal(views["k8"][bk].numpy(), pre["k_code"]), "K codes"
                vt = natural_key_order(views["vt8"][bk].numpy())
                assert np.array_equal(vt[:, :nk].T, pre["v_code"]), "V codes"
            # dS of this query head is over its key/value head's K
            ds = natural_key_order(views["ds"][bh].numpy())[:, :nk].astype(np.float64)
            ref = pre["qbar"].astype(np.float64) @ to_np64(kh).T
            scale = np.abs(pre["qbar"]).astype(np.float64) @ np.abs(to_np64(kh)).T + 1e-30
            assert np.max(np.abs(ds - ref) / scale) < 1e-5, "dS"


ATTN_CASES = [
    # name, B, H, H_kv, nq, nk, d, causal, layout, recipe
    ("g2_causal_d128", 1, 4, 2, 600, 600, 128, True, "HND", "llm"),
    ("g4_nhd_d64", 2, 8, 2, 300, 520, 64, False, "NHD", "video_dit"),
    ("mqa_causal_d64", 1, 6, 1, 333, 333, 64, True, "HND", "sweep"),
    ("g8_nhd_causal_d128", 1, 8, 1, 520, 300, 128, True, "NHD", "image_dit"),
    ("g3_d128", 1, 6, 2, 257, 700, 128, False, "HND", "image_dit"),
]


@pytest.mark.parametrize("name,B,H,Hk,nq,nk,d,causal,layout,recipe", ATTN_CASES, ids=[c[0] for c in ATTN_CASES])
def test_gqa_attention_matches_oracle(name, B, H, Hk, nq, nk, d, causal, layout, recipe):
    q, k, v = _inputs(B, H, Hk, nq, nk, d, causal, layout=layout, recipe=recipe)
    o = sage.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, layout=layout).cpu()
    assert o.shape == q.shape
    group = H // Hk
    for b in range(B):
        for h in range(H):
            qh, kh, vh = _head(q, b, h, layout), _head(k, b, h // group, layout), _head(v, b, h // group, layout)
            og = to_np64(_head(o, b, h, layout))
            _, oo = oracle_head(qh, kh, vh, causal=causal)
            assert_close_to_oracle(og, oo, "%s b%d h%d" % (name, b, h))
            ref = oracle.reference_attention(to_np64(qh)[None, None], to_np64(kh)[None, None],
                                             to_np64(vh)[None, None], causal=causal)[0, 0]
            assert cos(og, ref) >= O_COS_FULL


def test_gqa_equals_multi_head_on_repeated_kv_bit_exact():
    """The grouped call and the multi-head call on K, V with repeated heads compute the
    same codes and scales, so their outputs agree bit for bit."""
    B, H, Hk, n, d = 1, 8, 2, 700, 128
    q, k, v = (x.cuda() for x in _inputs(B, H, Hk, n, n, d, True))
    o_gqa = sage.attn_fwd(q, k, v, causal=True)
    rep = H // Hk
    o_mha = sage.attn_fwd(q, k.repeat_interleave(rep, dim=1).contiguous(), v.repeat_interleave(rep, dim=1).contiguous(),
                          causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o_gqa, o_mha)


def test_gqa_split_calls_equal_fused_call():
    B, H, Hk, nq, nk, d = 2, 4, 2, 333, 333, 64
    q, k, v = (x.cuda() for x in _inputs(B, H, Hk, nq, nk, d, True, recipe="video_dit"))
    o_full = sage.attn_fwd(q, k, v, causal=True)
    ws = sage.quant_qk(q, k)
    sage.quant_v(v, n_q=nq, workspace=ws)
    o_pre = sage.attn_fwd_prequant(ws, dtype=q.dtype, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o_full, o_pre)
    assert sage.get_device_status(ws) == (0, 0)


def test_gqa_bad_head_counts_rejected_before_launch():
    q = torch.zeros(1, 6, 128, 64, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 4, 128, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        sage.attn_fwd(q, k, k)
    lib = sage.load_library()
    o = torch.empty_like(q)
    ws = sage.make_workspace(1, 6, 128, 128, 64, H_kv=3)
    p = ctypes.c_void_p
    rc = lib.sage_attn_fwd_gqa(p(q.data_ptr()), p(k.data_ptr()), p(k.data_ptr()), p(o.data_ptr()), 1, 0, 1, 6, 4,
                               128, 128, 64, 0, 0.0, None, p(ws.ptr), ws.nbytes, None)
    assert rc == sage.SAGE_ERR_INVALID_ARG


def test_drop_in_interfaces_equal_attn_fwd():
    """SageAttention(...) and scaled_dot_product_attention(...) only marshal arguments:
    their outputs equal the attn_fwd call they stand for."""
    q, k, v = (x.cuda() for x in _inputs(1, 8, 2, 300, 300, 128, True))
    ref = sage.attn_fwd(q, k, v, causal=True)
    a = sage.SageAttention(head_dim=128, is_causal=True)
    assert torch.equal(a(q, k, v), ref)
    assert torch.equal(a(q, k, v), ref)   # the kept workspace is reused
    assert torch.equal(sage.scaled_dot_product_attention(q, k, v, is_causal=True, enable_gqa=True), ref)
    a16 = sage.SageAttention(head_dim=128, is_causal=True, quant_mode="qk_int8_pv_fp16", tensor_layout="NHD")
    qn, kn, vn = (x.transpose(1, 2).contiguous() for x in (q, k, v))
    assert torch.equal(a16(qn, kn, vn), sage.attn_fwd(qn, kn, vn, causal=True, layout="NHD", pv="fp16"))
