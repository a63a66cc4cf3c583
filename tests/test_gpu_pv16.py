"""The FP16 P / V mode ("qk_int8_pv_fp16") on the GPU, through the C ABI.

INT8 QK^T as in the default mode; P~ rounded to fp16 without the Pr scale, V rounded to
fp16 without a per-channel scale, PV on tcgen05 kind::f16 with FP32 accumulation.
Checked against the oracle's PV_FP16 mode, and for accuracy against full precision
next to the default FP8 mode.
"""
import numpy as np
import pytest
import torch

import oracle
import quantized_attention_fine_b200 as sage
from quantized_attention_fine_b200 import workloads as wl

from helpers import (O_COS_FULL, assert_close_to_oracle, cos, head_slices, natural_key_order, storage_positions,
                     to_np64)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from quantized_attention_fine_b200 import _build
    _build.build()
    sage.load_library()


def _inputs(name, B, H, Hk, nq, nk, d, causal, recipe, layout="HND", dtype=torch.bfloat16):
    w = wl.custom(name, B, H, nq, nk, d, causal, dtype=dtype, recipe=recipe, H_kv=Hk,
                  seed=9500 + nq + 3 * nk + d + 7 * H)
    q, k, v = wl.generate(w)
    if layout == "NHD":
        q, k, v = wl.to_nhd(q), wl.to_nhd(k), wl.to_nhd(v)
    return q, k, v


def test_fp16_v_prepass_bit_exact():
    B, H, nq, nk, d = 1, 2, 200, 300, 128
    q, k, v = _inputs("pv16_pre", B, H, H, nq, nk, d, False, "video_dit")
    mode = sage.QuantMode.make(pv="fp16")
    ws = sage.quant_qk(q.cuda(), k.cuda(), mode=mode)
    sage.quant_v(v.cuda(), n_q=nq, mode=mode, workspace=ws)
    torch.cuda.synchronize()
    vt = ws.view("vt8").cpu()
    assert vt.dtype == torch.float16
    for h in range(H):
        got = natural_key_order(vt[h].float().numpy().astype(np.float64))[:, :nk].T
        ref = oracle.f16_round(to_np64(v[0, h]).astype(np.float32))
        assert np.array_equal(got, ref)
        assert not natural_key_order(vt[h].float().numpy())[:, nk:].any()
        assert torch.all(ws.view("dv")[h].cpu() == 1.0)


CASES = [
    # name, B, H, H_kv, nq, nk, d, causal, layout, recipe, dtype
    ("d128_causal", 1, 2, 2, 600, 600, 128, True, "HND", "llm", torch.bfloat16),
    ("d64_full_nhd", 2, 2, 1, 300, 520, 64, False, "NHD", "video_dit", torch.bfloat16),
    ("d128_fp16_q_longer", 1, 4, 2, 520, 300, 128, True, "HND", "image_dit", torch.float16),
    ("d64_ragged", 1, 2, 2, 333, 333, 64, True, "HND", "sweep", torch.bfloat16),
]


@pytest.mark.parametrize("name,B,H,Hk,nq,nk,d,causal,layout,recipe,dtype", CASES, ids=[c[0] for c in CASES])
def test_pv16_matches_oracle_and_beats_fp8(name, B, H, Hk, nq, nk, d, causal, layout, recipe, dtype):
    q, k, v = _inputs(name, B, H, Hk, nq, nk, d, causal, recipe, layout, dtype)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o16, lse16 = sage.attn_fwd(qd, kd, vd, causal=causal, layout=layout, pv="fp16", return_lse=True)
    o8 = sage.attn_fwd(qd, kd, vd, causal=causal, layout=layout)
    o16, lse16, o8 = o16.cpu(), lse16.cpu().double().numpy(), o8.cpu()
    group = H // Hk
    err16, err8 = [], []
    for b in range(B):
        for h in range(H):
            qh = head_slices(q, q, q, b, h, layout)[0]
            kh, vh = head_slices(k, k, v, b, h // group, layout)[1:]
            pre = oracle.prepass_head(to_np64(qh), to_np64(kh), to_np64(vh), quant=oracle.PV_FP16)
            oo = oracle.attn_head(pre, causal=causal)
            og = to_np64(head_slices(o16, o16, o16, b, h, layout)[0])
            assert_close_to_oracle(og, oo, "%s b%d h%d" % (name, b, h))
            ll = oracle.lse_head(pre, causal=causal)
            fin = np.isfinite(ll)
            assert np.array_equal(np.isfinite(lse16[b, h]), fin)
            if fin.any():
                assert np.max(np.abs(lse16[b, h][fin] - ll[fin])) <= 1e-3
            ref = oracle.reference_attention(to_np64(qh)[None, None], to_np64(kh)[None, None],
                                             to_np64(vh)[None, None], causal=causal)[0, 0]
            if np.abs(ref).sum() > 0:
                assert cos(og, ref) >= O_COS_FULL
                err16.append(np.abs(og - ref).max())
                err8.append(np.abs(to_np64(head_slices(o8, o8, o8, b, h, layout)[0]) - ref).max())
    assert np.mean(err16) < np.mean(err8), (np.mean(err16), np.mean(err8))


def test_pv16_varlen_and_split_calls():
    lq = [300, 129, 0, 520]
    H, Hk, d = 4, 2, 128
    g = torch.Generator().manual_seed(9600)
    tq = sum(lq)
    q = torch.randn(tq, H, d, generator=g).to(torch.bfloat16)
    k = (torch.randn(tq, Hk, d, generator=g) + 2 * torch.randn(1, Hk, d, generator=g)).to(torch.bfloat16)
    v = torch.randn(tq, Hk, d, generator=g).to(torch.bfloat16)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lq)]), dtype=torch.int32)
    o = sage.attn_fwd_varlen(q.cuda(), k.cuda(), v.cuda(), cu.cuda(), cu.cuda(), causal=True, pv="fp16").cpu()
    oo = oracle.sage_attention_varlen(to_np64(q), to_np64(k), to_np64(v), cu.numpy(), cu.numpy(), causal=True,
                                      quant=oracle.PV_FP16)
    for b in range(len(lq)):
        s0, s1 = int(cu[b]), int(cu[b + 1])
        for h in range(H):
            if s1 > s0:
                assert_close_to_oracle(to_np64(o[s0:s1, h]), oo[s0:s1, h], "seq %d head %d" % (b, h))
    # split calls equal the fused call
    qd, kd, vd = (x.cuda() for x in _inputs("pv16_split", 2, 2, 2, 333, 333, 64, True, "video_dit"))
    mode = sage.QuantMode.make(pv="fp16")
    o_full = sage.attn_fwd(qd, kd, vd, causal=True, pv="fp16")
    ws = sage.quant_qk(qd, kd, mode=mode)
    sage.quant_v(vd, n_q=333, mode=mode, workspace=ws)
    o_pre = sage.attn_fwd_prequant(ws, dtype=qd.dtype, causal=True, mode=mode)
    torch.cuda.synchronize()
    assert torch.equal(o_full, o_pre)
    assert sage.get_device_status(ws) == (0, 0)


@pytest.mark.parametrize("nq,d,causal,H", [(8192, 128, True, 8), (4096, 64, False, 16)])
def test_pv16_long_sequences_deterministic(nq, d, causal, H):
    """The single P buffer per Q tile is reused every key tile: a race between its
    writers and the PV that reads it would show as run-to-run differences."""
    w = wl.custom("pv16_det", 1, H, nq, nq, d, causal, recipe="llm" if causal else "image_dit")
    q, k, v = (x.cuda() for x in wl.generate(w))
    mode = sage.QuantMode.make(pv="fp16")
    ws = sage.make_workspace(1, H, nq, nq, d, pv_fp16=True)
    sage.quant_qk(q, k, mode=mode, workspace=ws)
    sage.quant_v(v, n_q=nq, mode=mode, workspace=ws)
    outs = []
    for _ in range(3):
        o = torch.empty_like(q)
        sage.attn_fwd_prequant(ws, dtype=q.dtype, causal=causal, mode=mode, out=o)
        outs.append(o)
    torch.cuda.synchronize()
    assert sage.get_device_status(ws) == (0, 0)
    for o in outs[1:]:
        assert torch.equal(o, outs[0])
    # the last Q block of head 0 against the oracle
    pre = oracle.prepass_head(to_np64(q[0, 0].cpu()), to_np64(k[0, 0].cpu()), to_np64(v[0, 0].cpu()),
                              quant=oracle.PV_FP16)
    tq = nq // 128
    oo = oracle.attn_head(pre, causal=causal, qblocks=[tq - 1])
    rows = np.arange((tq - 1) * 128, nq)
    assert_close_to_oracle(to_np64(outs[0][0, 0].cpu())[rows], oo[rows], "last block")
