"""Q quantized inside the attention kernel (sage_attn_fwd_qfused_gqa), on the GPU.

This forward runs the K / V pre-pass and then an attention kernel that smooths and
quantizes its own Q tiles and forms the dS bias qbar . K of every key tile itself
("SageAttention2", arXiv 2411.10958, abstract: Q smoothed per 128-row block).  Checked
here:
  - the kernel's Q codes (written under the code-dump switch), delta_Q and qbar are
    bit-identical to the oracle's pre-pass, for every granularity, both dtypes and
    layouts, ragged tails and grouped-query heads;
  - the output and the LSE match the oracle on inputs whose Q has a channel bias (the
    workloads' Q has none, so there qbar and dS are near zero and would prove little);
  - the split entry (pre-pass + attention only) gives the whole forward's bits, and
    the pre-pass path's output up to the rounding of dS;
  - packed batches give the bits of one dense call per sequence;
  - rows that see no key, and Q smoothing switched off.
"""
import numpy as np
import pytest
import torch

import oracle
import quantized_attention_fine_b200 as sage
from quantized_attention_fine_b200 import workloads as wl

from helpers import GRAN_OF, assert_close_to_oracle, cos, head_slices, oracle_head, to_np64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from quantized_attention_fine_b200 import _build
    _build.build()
    sage.load_library()


def _inputs(B, H, H_kv, nq, nk, d, *, dtype=torch.bfloat16, layout="HND", q_bias=3.0, seed=0):
    """llm-recipe inputs plus a per-channel Q offset shared by every token of a head."""
    w = wl.custom("fq", B, H, nq, nk, d, False, dtype=dtype, recipe="llm", H_kv=H_kv,
                  seed=9100 + seed + 17 * H + 5 * nq + 3 * nk + d)
    q, k, v = wl.generate(w)
    g = torch.Generator().manual_seed(9200 + seed)
    q = (q.float() + q_bias * torch.randn((B, H, 1, d), generator=g)).to(dtype)
    if layout == "NHD":
        q, k, v = wl.to_nhd(q), wl.to_nhd(k), wl.to_nhd(v)
    return q, k, v


def _heads(B, H, H_kv):
    group = H // H_kv
    for b in range(B):
        for h in range(H):
            yield b, h, b * H + h, b * H_kv + h // group


CODE_CASES = [
    # B, H, H_kv, nq, nk, d, dtype, layout, granularity
    (1, 2, 2, 300, 520, 128, torch.bfloat16, "HND", "per_threadgroup"),
    (1, 2, 2, 256, 256, 64, torch.float16, "HND", "per_block"),
    (2, 3, 3, 200, 130, 128, torch.float16, "NHD", "per_warp"),
    (1, 4, 2, 333, 333, 64, torch.bfloat16, "NHD", "per_threadgroup"),
]


@pytest.mark.parametrize("B,H,Hk,nq,nk,d,dtype,layout,gran", CODE_CASES)
def test_in_kernel_q_codes_bit_exact(B, H, Hk, nq, nk, d, dtype, layout, gran):
    q, k, v = _inputs(B, H, Hk, nq, nk, d, dtype=dtype, layout=layout)
    ws = sage.make_workspace(B, H, nq, nk, d, device="cuda", H_kv=Hk)
    ws.tensor.fill_(0x5A)   # stale bytes: everything compared below must be written by the call
    off = ws.ptr - ws.tensor.data_ptr()
    ws.tensor[off:off + 256].zero_()   # but the status block starts clear
    sage.debug_set_q_code_dump(True)
    try:
        sage.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True, layout=layout, granularity=gran, workspace=ws,
                      fuse_q=True)
        torch.cuda.synchronize()
    finally:
        sage.debug_set_q_code_dump(False)
    views = {n: ws.view(n).cpu() for n in ("q8", "dq", "qbar")}
    g_q, g_k = GRAN_OF[gran]
    for b, h, bh, _ in _heads(B, H, Hk):
        hk = h // (H // Hk)
        qh = q[b, h] if layout == "HND" else q[b, :, h]
        kh, vh = (x[b, hk] if layout == "HND" else x[b, :, hk] for x in (k, v))
        pre = oracle.prepass_head(to_np64(qh), to_np64(kh), to_np64(vh), g_q=g_q, g_k=g_k)
        assert np.array_equal(views["qbar"][bh].numpy(), pre["qbar"]), "qbar, head %d" % bh
        assert np.array_equal(views["dq"][bh].numpy(), pre["dq_row"]), "delta_Q, head %d" % bh
        got = views["q8"][bh].numpy()
        assert np.array_equal(got, pre["q_code"]), "Q codes, head %d: %d of %d differ" % (
            bh, int((got != pre["q_code"]).sum()), got.size)
    assert sage.get_device_status(ws) == (0, 0)


BIAS_CASES = [
    # name, B, H, nq, nk, d, causal, layout, dtype
    ("d128_causal", 1, 2, 520, 520, 128, True, "HND", torch.bfloat16),
    ("d128_cross", 1, 2, 300, 700, 128, False, "NHD", torch.float16),
    ("d64_causal", 2, 2, 333, 333, 64, True, "HND", torch.float16),
    ("d64_full", 1, 3, 256, 640, 64, False, "NHD", torch.bfloat16),
]


@pytest.mark.parametrize("name,B,H,nq,nk,d,causal,layout,dtype", BIAS_CASES)
def test_q_bias_output_and_lse_match_oracle(name, B, H, nq, nk, d, causal, layout, dtype):
    q, k, v = _inputs(B, H, H, nq, nk, d, dtype=dtype, layout=layout, q_bias=4.0, seed=1)
    o, lse = sage.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, layout=layout, return_lse=True, fuse_q=True)
    torch.cuda.synchronize()
    o, lse = o.cpu(), lse.cpu()
    for b in range(B):
        for h in range(H):
            qh, kh, vh = head_slices(q, k, v, b, h, layout)
            pre, oo = oracle_head(qh, kh, vh, causal=causal)
            og = o[b, h] if layout == "HND" else o[b, :, h]
            assert_close_to_oracle(to_np64(og), oo, "%s b%d h%d" % (name, b, h))
            ref = oracle.lse_head(pre, causal=causal)
            got = lse[b, h].double().numpy()
            fin = np.isfinite(ref)
            assert np.array_equal(np.isfinite(got), fin)
            assert np.max(np.abs(got[fin] - ref[fin])) <= 1e-3, name


def test_q_bias_is_taken_out_by_smoothing():
    """With a large Q channel offset the smoothed path stays as close to full-precision
    attention as without one: the offset's share of the scores goes through dS."""
    B, H, n, d = 1, 2, 512, 128
    errs = []
    for bias in (0.0, 8.0):
        q, k, v = _inputs(B, H, H, n, n, d, q_bias=bias, seed=2)
        o = sage.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True, fuse_q=True).cpu()
        full = oracle.reference_attention(to_np64(q), to_np64(k), to_np64(v), causal=True)
        errs.append(cos(to_np64(o), full))
    assert min(errs) >= 0.999, errs


def test_split_entry_gives_the_whole_forward_bits():
    B, H, Hk, nq, nk, d = 2, 4, 2, 333, 333, 64
    q, k, v = (x.cuda() for x in _inputs(B, H, Hk, nq, nk, d, dtype=torch.float16, seed=3))
    o_full = sage.attn_fwd(q, k, v, causal=True, fuse_q=True)
    ws = sage.quant_qk(q, k)
    sage.quant_v(v, n_q=nq, workspace=ws)
    o_split = sage.attn_fwd_qfused(q, k, ws, causal=True)
    o_pre = sage.attn_fwd_prequant(ws, dtype=q.dtype, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o_full, o_split)
    # the pre-pass path differs only in the rounding of dS (a different summation order)
    err = (o_full.double() - o_pre.double()).abs().max().item()
    assert err <= 1e-2, err
    assert cos(o_full.cpu().double().numpy(), o_pre.cpu().double().numpy()) >= 0.99999
    assert sage.get_device_status(ws) == (0, 0)


def test_packed_batch_matches_dense_calls():
    H, Hk, d = 4, 2, 128
    lens_q, lens_kv = [130, 1, 300], [200, 77, 300]
    g = torch.Generator().manual_seed(9300)
    qs = [(torch.randn(n, H, d, generator=g) + 3.0 * torch.randn(1, H, d, generator=g)).bfloat16() for n in lens_q]
    ks = [torch.randn(n, Hk, d, generator=g).bfloat16() for n in lens_kv]
    vs = [torch.randn(n, Hk, d, generator=g).bfloat16() for n in lens_kv]
    q, k, v = (torch.cat(x).cuda() for x in (qs, ks, vs))
    cu_q = torch.tensor(np.cumsum([0] + lens_q), dtype=torch.int32, device="cuda")
    cu_kv = torch.tensor(np.cumsum([0] + lens_kv), dtype=torch.int32, device="cuda")
    o = sage.attn_fwd_varlen(q, k, v, cu_q, cu_kv, causal=True, fuse_q=True)
    torch.cuda.synchronize()
    for i in range(len(lens_q)):
        ref = sage.attn_fwd(qs[i][None].cuda(), ks[i][None].cuda(), vs[i][None].cuda(), causal=True, layout="NHD",
                            fuse_q=True)[0]
        torch.cuda.synchronize()
        assert torch.equal(o[int(cu_q[i]):int(cu_q[i + 1])], ref), "sequence %d" % i


def test_rows_without_keys_and_no_q_smoothing():
    B, H, nq, nk, d = 1, 2, 520, 150, 128   # causal, bottom-right: the first 370 rows see no key
    q, k, v = _inputs(B, H, H, nq, nk, d, seed=4)
    for smooth_q in (True, False):
        o = sage.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True, smooth_q=smooth_q, fuse_q=True).cpu()
        for h in range(H):
            _, oo = oracle_head(q[0, h], k[0, h], v[0, h], causal=True, smooth_q=smooth_q)
            assert_close_to_oracle(to_np64(o[0, h]), oo, "smooth_q=%s h%d" % (smooth_q, h))
        assert torch.count_nonzero(o[:, :, :nq - nk]) == 0


@pytest.mark.parametrize("d", [64, 128])
def test_fp16_pv_mode(d):
    """The qk_int8_pv_fp16 mode with Q quantized in the kernel, against the oracle's
    PV_FP16 mode."""
    B, H, nq, nk = 1, 2, 300, 450
    q, k, v = _inputs(B, H, H, nq, nk, d, q_bias=3.0, seed=5)
    o = sage.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True, pv="fp16", fuse_q=True).cpu()
    for h in range(H):
        pre = oracle.prepass_head(to_np64(q[0, h]), to_np64(k[0, h]), to_np64(v[0, h]), quant=oracle.PV_FP16)
        oo = oracle.attn_head(pre, causal=True)
        assert_close_to_oracle(to_np64(o[0, h]), oo, "pv16 d%d h%d" % (d, h))


def test_four_bit_mode_is_refused():
    q, k, v = (x.cuda() for x in _inputs(1, 1, 1, 128, 128, 64, seed=6))
    with pytest.raises(sage.SageError):
        sage.attn_fwd(q, k, v, granularity="fp4", fuse_q=True)


@pytest.mark.parametrize("d", [64, 128])
def test_bounded_waits_report_timeout_and_context_survives(d):
    """One K slot's signal withheld: the kernel that quantizes Q itself leaves through its
    bounded waits (Q quantization, dS warp, producers, MMA issuer), records the timeout,
    and the context stays usable.  Eight key tiles, so that the dS warp also meets a
    K-stage wait that never completes."""
    q, k, v = (x.cuda() for x in _inputs(1, 1, 1, 256, 1024, d, seed=7))
    ws = sage.quant_qk(q, k)
    sage.quant_v(v, n_q=256, workspace=ws)
    assert sage.get_device_status(ws) == (0, 0)
    out = torch.zeros_like(q)
    sage.debug_fault_inject_qfused(q, k, ws, out)
    code, site = sage.get_device_status(ws)
    assert code == sage.SAGE_ERR_TIMEOUT and site != 0
    assert sage.get_device_status(ws) == (0, 0)
    o = sage.attn_fwd_qfused(q, k, ws).cpu()
    torch.cuda.synchronize()
    assert sage.get_device_status(ws) == (0, 0)
    _, oo = oracle_head(q[0, 0].cpu(), k[0, 0].cpu(), v[0, 0].cpu(), causal=False)
    assert_close_to_oracle(to_np64(o[0, 0]), oo, "after timeout")
