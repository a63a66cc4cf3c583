"""Parity at the full workload sizes, in the launch configuration bench.py times
(sage_quant_qk + sage_quant_v + sage_attn_fwd_prequant on one workspace), and for
llm_prefill also through the path with Q quantized inside the attention kernel
(sage_attn_fwd_qfused_gqa, `bench.py --fuse-q`; its Q codes read back through the
code-dump switch).

The oracle cannot redo a whole 32K-token workload, so it recomputes sampled heads
completely (pre-pass, bit-exact) and sampled Q blocks of them over the full KV range
(attention output within tolerance); full-precision attention is evaluated on the
same rows in numpy fp64.
"""
import numpy as np
import pytest
import torch

import oracle
import quantized_attention_fine_b200 as sage
from quantized_attention_fine_b200 import workloads as wl

from helpers import O_COS_FULL, assert_close_to_oracle, cos, natural_key_order, rows_of_blocks, to_np64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from quantized_attention_fine_b200 import _build
    _build.build()
    sage.load_library()


def _full_precision_rows(qh, kh, vh, rows, causal):
    q = qh[rows]
    x = (q @ kh.T) / np.sqrt(qh.shape[1])
    if causal:
        off = kh.shape[0] - qh.shape[0]
        j = np.arange(kh.shape[0])[None, :]
        x = np.where(j <= rows[:, None] + off, x, -np.inf)
    m = x.max(1, keepdims=True)
    p = np.exp(x - m)
    return (p @ vh) / p.sum(1, keepdims=True)


@pytest.mark.parametrize("name,path", [("image_dit", "prequant"), ("llm_prefill", "prequant"),
                                       ("video_dit", "prequant"), ("llm_prefill_gqa", "prequant"),
                                       ("sweep_n65536_d128_causal", "prequant"), ("sweep_n65536_d64_full", "prequant"),
                                       ("llm_prefill", "fuse_q")])
def test_full_size_workload_sampled(name, path):
    """Also the longest sweep points, N = 65,536 (the sweep recipe names N up to 64K):
    the first, middle and last Q blocks of two heads over all 65,536 keys."""
    w = wl.by_name(name)
    q, k, v = wl.generate(w)
    dev = torch.device("cuda", 0)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    mode = sage.QuantMode.make()
    ws = sage.make_workspace(w.B, w.H, w.N_q, w.N_kv, w.d, device=dev, H_kv=w.Hk)
    if path == "fuse_q":
        sage.debug_set_q_code_dump(True)
        try:
            o = sage.attn_fwd(qd, kd, vd, causal=w.causal, workspace=ws, fuse_q=True)
            torch.cuda.synchronize()
        finally:
            sage.debug_set_q_code_dump(False)
    else:
        sage.quant_qk(qd, kd, mode=mode, workspace=ws)
        sage.quant_v(vd, n_q=w.N_q, mode=mode, workspace=ws)
        o = sage.attn_fwd_prequant(ws, dtype=q.dtype, causal=w.causal, mode=mode)
    assert sage.get_device_status(ws) == (0, 0)
    tq = -(-w.N_q // 128)
    heads = [(0, 0), (w.B - 1, w.H - 1)]
    group = w.H // w.Hk
    blocks = sorted({0, tq // 2, tq - 1})
    views = {n: ws.view(n) for n in ("q8", "k8", "vt8", "dq", "dk", "dv", "qbar", "kbar")}
    for b, h in heads:
        bh, bk = b * w.H + h, b * w.Hk + h // group   # query head, its key/value head
        qh, kh, vh = to_np64(q[b, h]), to_np64(k[b, h // group]), to_np64(v[b, h // group])
        pre = oracle.prepass_head(qh, kh, vh)
        # the pre-pass of the sampled head, bit-exact
        assert np.array_equal(views["qbar"][bh].cpu().numpy(), pre["qbar"])
        assert np.array_equal(views["kbar"][bk].cpu().numpy(), pre["kbar"])
        assert np.array_equal(views["dq"][bh].cpu().numpy(), pre["dq_row"])
        assert np.array_equal(views["dk"][bk].cpu().numpy(), pre["dk_key"][::16])
        assert np.array_equal(views["dv"][bk].cpu().numpy(), pre["dv"])
        assert np.array_equal(views["q8"][bh].cpu().numpy(), pre["q_code"])
        assert np.array_equal(views["k8"][bk].cpu().numpy(), pre["k_code"])
        assert np.array_equal(natural_key_order(views["vt8"][bk].cpu().numpy())[:, :w.N_kv].T, pre["v_code"])
        # attention rows of the sampled Q blocks over the full KV range
        oo = oracle.attn_head(pre, causal=w.causal, qblocks=blocks)
        rows = rows_of_blocks(w.N_q, blocks)
        og = to_np64(o[b, h].cpu())[rows]
        assert_close_to_oracle(og, oo[rows], "%s head (%d,%d)" % (name, b, h))
        ref = _full_precision_rows(qh, kh, vh, rows, w.causal)
        assert cos(og, ref) >= O_COS_FULL, "%s: cos vs full precision %.5f" % (name, cos(og, ref))
        # the rows' log-sum-exp of the same blocks
        ll = oracle.lse_head(pre, causal=w.causal, qblocks=blocks)
        lg = ws.lse()[b, h].cpu().double().numpy()[rows]
        assert np.max(np.abs(lg - ll[rows])) <= 1e-3, "%s: LSE" % name


def test_full_size_fp16_pv_mode_sampled():
    """The FP16 P / V mode at the llm_prefill size, in the launch configuration of
    `bench.py --pv fp16`: sampled heads and Q blocks against the oracle's PV_FP16 mode."""
    w = wl.LLM_PREFILL
    q, k, v = wl.generate(w)
    dev = torch.device("cuda", 0)
    ws = sage.make_workspace(w.B, w.H, w.N_q, w.N_kv, w.d, device=dev, pv_fp16=True)
    o = sage.attn_fwd(q.to(dev), k.to(dev), v.to(dev), causal=True, pv="fp16", workspace=ws)
    assert sage.get_device_status(ws) == (0, 0)
    tq = w.N_q // 128
    blocks = [0, tq // 2, tq - 1]
    rows = rows_of_blocks(w.N_q, blocks)
    for h in (0, w.H - 1):
        qh, kh, vh = to_np64(q[0, h]), to_np64(k[0, h]), to_np64(v[0, h])
        pre = oracle.prepass_head(qh, kh, vh, quant=oracle.PV_FP16)
        oo = oracle.attn_head(pre, causal=True, qblocks=blocks)
        og = to_np64(o[0, h].cpu())[rows]
        assert_close_to_oracle(og, oo[rows], "pv16 head %d" % h)
        assert cos(og, _full_precision_rows(qh, kh, vh, rows, True)) >= O_COS_FULL


def test_full_size_fp4_video_dit_sampled():
    """The 4-bit mode at the video_dit size (B2 H48 N17776 d64, the d = 64 workload it
    runs on), in the launch configuration of `bench.py --qk fp4`: sampled heads and Q
    blocks against the oracle's FP4 mode, and against full precision."""
    w = wl.VIDEO_DIT
    q, k, v = wl.generate(w)
    dev = torch.device("cuda", 0)
    mode = sage.QuantMode.make("fp4")
    ws = sage.make_workspace(w.B, w.H, w.N_q, w.N_kv, w.d, device=dev, qk_fp4=True)
    sage.quant_qk(q.to(dev), k.to(dev), mode=mode, workspace=ws)
    sage.quant_v(v.to(dev), n_q=w.N_q, mode=mode, workspace=ws)
    o = sage.attn_fwd_prequant(ws, dtype=q.dtype, causal=w.causal, mode=mode)
    assert sage.get_device_status(ws) == (0, 0)
    tq = -(-w.N_q // 128)
    blocks = [0, tq // 2, tq - 1]
    rows = rows_of_blocks(w.N_q, blocks)
    for b, h in ((0, 0), (w.B - 1, w.H - 1)):
        qh, kh, vh = to_np64(q[b, h]), to_np64(k[b, h]), to_np64(v[b, h])
        pre = oracle.prepass_head(qh, kh, vh, quant=oracle.QK_FP4_PV_FP8)
        oo = oracle.attn_head(pre, causal=False, qblocks=blocks)
        og = to_np64(o[b, h].cpu())[rows]
        assert_close_to_oracle(og, oo[rows], "fp4 video_dit head (%d,%d)" % (b, h))
        # FP4 is the lossier mode: the oracle's own FP4 cosine on this workload is 0.9896
        assert cos(og, _full_precision_rows(qh, kh, vh, rows, False)) >= 0.98
