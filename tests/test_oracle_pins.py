"""Pins of the fp64 oracle to facts outside itself (no GPU needed).

Each test ties one oracle step to a closed form, an invariant, a library routine,
a brute-force computation on tiny inputs, or a number printed on the pages
(tests/golden/page_constants.json).  A plausible slip in the oracle (a dropped
dS term, a wrong sign, a transposed operand, a wrong scale in the epilogue, a
mis-rounded code) fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from quantized_attention_fine_b200 import workloads as wl

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_constants.json")))


def _rand_head(nq, nk, d, seed, kbias=3.0, qbias=0.0, outliers=True, dtype=torch.bfloat16):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(nq, d, generator=g) + qbias * torch.randn(1, d, generator=g)
    k = torch.randn(nk, d, generator=g) + kbias * torch.randn(1, d, generator=g)
    v = torch.randn(nk, d, generator=g)
    if outliers:
        m = torch.rand(nq, d, generator=g) < 0.01
        q = torch.where(m, q * 20, q)
    return (q.to(dtype).double().numpy(), k.to(dtype).double().numpy(), v.to(dtype).double().numpy())


def _textbook(q, k, v, causal, scale):
    """Full-precision softmax attention in numpy fp64 (independent of the C oracle)."""
    nq, nk = q.shape[0], k.shape[0]
    x = (q @ k.T) * scale
    if causal:
        i = np.arange(nq)[:, None]
        j = np.arange(nk)[None, :]
        x = np.where(j <= i + (nk - nq), x, -np.inf)
    m = np.max(x, axis=1, keepdims=True)
    out = np.zeros((nq, v.shape[1]))
    ok = np.isfinite(m[:, 0])
    p = np.exp(x[ok] - m[ok])
    out[ok] = (p @ v) / p.sum(axis=1, keepdims=True)
    return out


# ---------------------------------------------------------------------------
# E4M3 codec
# ---------------------------------------------------------------------------
def test_e4m3_decode_all_codes_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan_ours, nan_ref = np.isnan(ours), np.isnan(ref)
    assert (nan_ours == nan_ref).all() and nan_ref.sum() == 2  # 0x7F, 0xFF
    assert np.array_equal(ours[~nan_ref], ref[~nan_ref])
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9


def test_e4m3_encode_matches_torch_in_range():
    g = torch.Generator().manual_seed(7)
    parts = [
        torch.randn(20000, generator=g) * 50,
        torch.rand(20000, generator=g) * 2.0 ** -6,            # subnormal range
        torch.exp2(torch.randint(-12, 9, (4000,), generator=g).float()) * (1 + torch.randint(0, 16, (4000,), generator=g).float() / 16),  # ties
        torch.tensor([0.0, -0.0, 448.0, -448.0, 464.0, -464.0, 2.0 ** -10, 3 * 2.0 ** -10, 2.0 ** -6]),
    ]
    x = torch.cat(parts).float()
    x = x[x.abs() <= 464.0]
    ours = oracle.e4m3_encode(x.numpy())
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_e4m3_saturates_to_448():
    # satfinite: every finite value beyond the largest code maps to +-448
    x = np.array([465.0, 480.0, 1e4, 3e38, -500.0], dtype=np.float32)
    assert list(oracle.e4m3_encode(x)) == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE]


def test_page_pr_vr_values_exact_in_e4m3_and_within_bound():
    """Pr = 224 / Vr = 4.5 and the other printed pairs are E4M3 values whose product stays
    within the printed FP16-accumulator bound Pr x Vr <= 2047/2 (derived from |32 p v| <= 65504
    with one more FP16 accumulation)."""
    bound = GOLDEN["pr_vr_bound"]["value"]
    # |32 p v| <= 65504 per mma, two mma results summed in FP16: 64 Pr Vr <= 65504
    assert bound == GOLDEN["fp16_max"]["value"] / 64 == 2047 / 2
    for pr, vr in GOLDEN["pr_vr_alternatives"]["value"]:
        p8 = oracle.e4m3_decode(oracle.e4m3_encode([pr]))[0]
        v8 = oracle.e4m3_decode(oracle.e4m3_encode([vr]))[0]
        assert p8 == pr and v8 == vr
        assert p8 * v8 <= bound
    assert GOLDEN["e4m3_max"]["value"] == oracle.e4m3_decode([0x7E])[0]


@pytest.mark.parametrize("vr_key,divisor", [("vr_sa2pp", 2304.0), ("vr_sa2", 448.0 * 512.0)])
def test_v_underflow_threshold_from_pages(vr_key, divisor):
    """Per-channel V scaling: an entry of size colmax / (Vr 2^9) lands exactly on the smallest
    E4M3 subnormal, one below half of it flushes to 0.  For Vr = 4.5 the divisor is the
    printed 2304; for Vr = 448 it is 448 * 2^9 (printed as ~229k)."""
    vr = GOLDEN[vr_key]["value"]
    if vr_key == "vr_sa2pp":
        assert divisor == GOLDEN["underflow_divisor_vr_4_5"]["value"]
        assert abs(vr * 512 - GOLDEN["dynamic_range_vr_4_5_approx"]["value"]) < 50
    else:
        assert abs(divisor - GOLDEN["dynamic_range_vr_448_approx"]["value"]) < 1000
    colmax = 3.0
    col = np.array([colmax, colmax / divisor, 0.49 * colmax / divisor, -colmax / divisor, 0.0])
    nk = col.size
    v = np.zeros((nk, 2))
    v[:, 0] = col
    v[:, 1] = 1.0
    q = np.zeros((1, 2))
    k = np.zeros((nk, 2))
    pre = oracle.prepass_head(q, k, v, v_range=vr)
    codes = pre["v_code"][:, 0]
    assert codes[0] == oracle.e4m3_encode([vr])[0]
    assert codes[1] == 0x01 and codes[3] == 0x81
    assert codes[2] == 0x00 and codes[4] == 0x00


# ---------------------------------------------------------------------------
# INT8 quantization
# ---------------------------------------------------------------------------
def test_int8_code_matches_torch_round_half_even():
    g = torch.Generator().manual_seed(3)
    xs = (torch.randn(50000, generator=g) * 3).float()
    delta = torch.full_like(xs, float(np.float32(2.9) / np.float32(127)))
    xs[:9] = torch.tensor([0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 126.5, 127.49, -200.0]) * delta[:9]
    ours = oracle.int8_code(xs.numpy(), delta.numpy())
    ref = torch.clamp(torch.round(xs / delta), -127, 127).to(torch.int8).numpy()
    assert np.array_equal(ours, ref)


@pytest.mark.parametrize("gran", ["per_block", "per_warp", "per_threadgroup"])
def test_int8_codes_residual_bound_and_group_extremes(gran):
    g_q, g_k = oracle.GRANULARITY[gran]
    q, k, v = _rand_head(200, 300, 64, seed=11)
    pre = oracle.prepass_head(q, k, v, g_q=g_q, g_k=g_k)
    nq, nk = 200, 300
    # smoothed fp32 values exactly as the quantizer sees them
    qb = np.repeat(pre["qbar"], 128, axis=0)[:nq]
    xs_q = (q.astype(np.float32) - qb).astype(np.float32)
    xs_k = (k.astype(np.float32) - pre["kbar"][None, :]).astype(np.float32)
    for xs, code, dl, G in ((xs_q, pre["q_code"][:nq], pre["dq_row"][:nq], g_q),
                            (xs_k, pre["k_code"][:nk], pre["dk_key"][:nk], g_k)):
        quot = xs / dl[:, None]
        assert np.all(np.abs(quot - code) <= 0.5 + 1e-5)          # round to nearest
        assert np.abs(code).max() <= 127
        # scale constant on each group, and each group's amax maps to +-127
        n = xs.shape[0]
        for g0 in range(0, n, G):
            rows = slice(g0, min(g0 + G, n))
            assert len(set(dl[rows].tolist())) == 1
            amax = np.abs(xs[rows]).max()
            if amax > 0:
                assert dl[g0] == np.float32(amax) / np.float32(127)
                assert np.abs(code[rows]).max() == 127
    # elementwise bound on the dequantized scores
    ks = pre["k_s"]
    qs = q - qb.astype(np.float64)
    s_true = qs @ ks.T
    s_deq = (pre["dq_row"][:nq, None] * pre["q_code"][:nq].astype(np.float64)) @ \
            (pre["dk_key"][:nk, None] * pre["k_code"][:nk].astype(np.float64)).T
    dq = pre["dq_row"][:nq, None].astype(np.float64)
    dk = pre["dk_key"][None, :nk].astype(np.float64)
    bound = (dq / 2) * np.abs(ks).sum(1)[None, :] + (dk / 2) * np.abs(qs).sum(1)[:, None] + dq * dk / 4 * 64
    assert np.all(np.abs(s_deq - s_true) <= bound * (1 + 1e-6) + 1e-9)


def test_integer_scores_exact_against_int64_matmul():
    q, k, v = _rand_head(128, 256, 128, seed=5)
    pre = oracle.prepass_head(q, k, v)
    s_int = pre["q_code"].astype(np.int64) @ pre["k_code"].astype(np.int64).T
    assert np.abs(s_int).max() < 2 ** 31
    # the oracle's attention multiplies q_hat . k_hat: integer-valued doubles
    assert np.array_equal(pre["q_hat"] @ pre["k_hat"].T, s_int.astype(np.float64))


# ---------------------------------------------------------------------------
# Smoothing identities
# ---------------------------------------------------------------------------
def test_q_smoothing_identity_exact():
    """(Q - qbar) K_s^T + dS = Q K_s^T, and Q K_s^T differs from Q K^T by a per-row constant."""
    q, k, v = _rand_head(300, 260, 64, seed=21, qbias=2.0)
    pre = oracle.prepass_head(q, k, v, quant=(0, 1, 1))
    nq = 300
    for t in range(3):
        rows = slice(128 * t, min(128 * t + 128, nq))
        lhs = pre["q_hat"][rows] @ pre["k_s"].T + oracle.delta_s(pre, t)[None, :]
        rhs = q[rows] @ pre["k_s"].T
        assert np.max(np.abs(lhs - rhs)) < 1e-11
        diff = q[rows] @ k.T - rhs
        assert np.max(np.abs(diff - diff[:, :1])) < 1e-11


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("nq,nk", [(256, 256), (200, 333), (333, 200), (1, 129), (130, 1)])
def test_quant_off_equals_textbook_attention(causal, nq, nk):
    """With every quantizer set to identity the method is exact attention: the smoothing
    (K mean, Q block mean + dS) and the tiled online softmax cancel exactly."""
    q, k, v = _rand_head(nq, nk, 64, seed=nq * 7 + nk, qbias=1.5)
    pre = oracle.prepass_head(q, k, v, quant=(0, 0, 0), smooth_q=True, smooth_k=True)
    o = oracle.attn_head(pre, causal=causal)
    ref = _textbook(q, k, v, causal, 1 / 8)
    assert np.max(np.abs(o - ref)) < 1e-12
    ref_c = oracle.reference_attention(q[None, None], k[None, None], v[None, None], causal=causal)[0, 0]
    assert np.max(np.abs(ref_c - ref)) < 1e-12


def test_k_smoothing_invariance_without_quantization():
    q, k, v = _rand_head(256, 384, 64, seed=31, kbias=10.0)
    a = oracle.attn_head(oracle.prepass_head(q, k, v, quant=(0, 0, 0), smooth_k=True, smooth_q=False))
    b = oracle.attn_head(oracle.prepass_head(q, k, v, quant=(0, 0, 0), smooth_k=False, smooth_q=False))
    assert np.max(np.abs(a - b)) < 1e-12


def test_smoothing_improves_int8_accuracy_with_channel_bias():
    """The point of smoothing: with a large per-channel K bias, INT8 QK without K smoothing is
    much worse than with it (relative to textbook attention)."""
    q, k, v = _rand_head(256, 512, 64, seed=41, kbias=20.0)
    ref = _textbook(q, k, v, False, 1 / 8)

    def err(**kw):
        o = oracle.attn_head(oracle.prepass_head(q, k, v, quant=(1, 0, 0), **kw))
        return np.abs(o - ref).mean()
    assert err(smooth_k=True, smooth_q=True) < 0.5 * err(smooth_k=False, smooth_q=False)


# ---------------------------------------------------------------------------
# FP8 P and V
# ---------------------------------------------------------------------------
def test_v_quantization_only_equals_attention_on_dequantized_v():
    q, k, v = _rand_head(256, 300, 64, seed=51)
    pre = oracle.prepass_head(q, k, v, quant=(0, 0, 1))
    v_deq = pre["v_hat"] * pre["dv"][None, :].astype(np.float64)
    rel = np.abs(v_deq - v) / np.maximum(np.abs(v), 1e-30)
    normal = np.abs(v) / pre["dv"][None, :] >= 2.0 ** -6
    assert rel[normal].max() <= 2.0 ** -4 + 1e-12           # half an E4M3 ulp
    o = oracle.attn_head(pre)
    ref = _textbook(q, k, v_deq, False, 1 / 8)
    assert np.max(np.abs(o - ref)) < 1e-12


def test_p_quantization_with_max_in_first_tile_equals_two_pass():
    """If every row's maximum logit sits in the first KV tile, the running max never changes,
    so the tiled E4M3 rounding of P~ Pr equals a two-pass computation with the final max."""
    nq, nk, d = 128, 384, 64
    q, k, v = _rand_head(nq, nk, d, seed=61, outliers=False)
    q[:, 0] = 1.0
    k[:, 0] = 0.0
    x0 = (q @ k.T) / 8.0
    margin = np.max(x0[:, 128:].max(1) - x0[:, 5]) + 2.0
    k[5, 0] = 8.0 * margin                              # key 5 (tile 0) wins every row by >= 2
    pr = 448.0
    pre = oracle.prepass_head(q, k, v, quant=(0, 1, 0), smooth_q=False, smooth_k=False)
    o = oracle.attn_head(pre)
    x = (q @ k.T) / 8.0
    assert np.all(np.argmax(x, axis=1) < 128)
    m = x.max(1, keepdims=True)
    p = np.exp(x - m)
    assert (p[:, 128:] > 2.0 ** -9 / pr).mean() > 0.5    # later tiles still contribute
    p8 = torch.from_numpy(p * pr).float().to(torch.float8_e4m3fn).to(torch.float64).numpy()
    ref = (p8 @ (pre["v_hat"] * pre["dv"][None, :])) / pr / p.sum(1, keepdims=True)
    assert np.max(np.abs(o - ref)) < 1e-12


def test_full_method_brute_force_tiny():
    """Independent brute force on a tiny head with library codecs (torch.round, float8_e4m3fn),
    vectorised per KV tile, against the oracle's loop nest."""
    nq, nk, d, causal = 200, 300, 64, True
    q, k, v = _rand_head(nq, nk, d, seed=71)
    pre = oracle.prepass_head(q, k, v, g_q=32, g_k=16)
    o = oracle.attn_head(pre, causal=causal)

    T = torch
    qt, kt, vt = T.from_numpy(q), T.from_numpy(k), T.from_numpy(v)
    tq = -(-nq // 128)
    qpad = T.zeros(tq * 128, d, dtype=T.float64)
    qpad[:nq] = qt
    qbar = T.stack([qt[128 * t:min(128 * t + 128, nq)].mean(0) for t in range(tq)]).float()
    valid = T.arange(tq * 128) < nq
    xs_q = T.where(valid[:, None], qpad.float() - qbar.repeat_interleave(128, 0), T.zeros(()))
    dq = xs_q.abs().reshape(-1, 32, d).amax(dim=(1, 2)).float() / 127.0
    dq = T.where(dq == 0, T.ones(()), dq).repeat_interleave(32)
    cq = T.clamp(T.round(xs_q / dq[:, None]), -127, 127).to(T.int64)
    kbar = kt.mean(0).float()
    nk_pad = -(-nk // 128) * 128
    xs_k = T.zeros(nk_pad, d)
    xs_k[:nk] = kt.float() - kbar
    dk = xs_k.abs().reshape(-1, 16, d).amax(dim=(1, 2)) / 127.0
    dk = T.where(dk == 0, T.ones(()), dk).repeat_interleave(16)
    ck = T.clamp(T.round(xs_k / dk[:, None]), -127, 127).to(T.int64)
    s = (dq[:, None].double() * dk[None, :].double()) * (cq @ ck.T).double()
    ks64 = kt - kbar.double()
    ds = qbar.double() @ ks64.T
    s = s[:nq, :nk] + ds.repeat_interleave(128, 0)[:nq]
    x = s / 8.0
    i = T.arange(nq)[:, None]
    j = T.arange(nk)[None, :]
    x = T.where(j <= i + (nk - nq), x, T.tensor(-float("inf"), dtype=T.float64))
    dv = vt.abs().amax(0).float() / 448.0
    v8 = (vt.float() / dv).to(T.float8_e4m3fn).double()
    m = T.full((nq, 1), -float("inf"), dtype=T.float64)
    l = T.zeros(nq, 1, dtype=T.float64)
    acc = T.zeros(nq, d, dtype=T.float64)
    for j0 in range(0, nk, 128):
        xt = x[:, j0:j0 + 128]
        mt = T.maximum(m, xt.amax(1, keepdim=True))
        seen = T.isfinite(mt)
        alpha = T.where(T.isfinite(m), T.exp(m - mt), T.zeros(()))
        alpha = T.where(seen, alpha, T.ones(()))
        p = T.where(seen, T.exp(xt - T.where(seen, mt, T.zeros(()))), T.zeros(()))
        l = alpha * l + p.sum(1, keepdim=True)
        p8 = (p * 448.0).float().to(T.float8_e4m3fn).double()
        acc = alpha * acc + p8 @ v8[j0:j0 + 128]
        m = T.where(seen, mt, m)
    ref = T.where(l > 0, acc / 448.0 * dv.double() / T.where(l > 0, l, T.ones(())), T.zeros(()))
    assert np.array_equal(pre["q_code"], cq.to(T.int8).numpy())
    assert np.array_equal(pre["k_code"], ck.to(T.int8).numpy())
    assert np.max(np.abs(o - ref.numpy())) < 1e-12


def test_causal_rows_ignore_future_keys():
    """Replacing every operand of keys >= cut (codes, smoothed K, V) leaves rows < cut unchanged."""
    nq = nk = 300
    cut = 150
    q, k, v = _rand_head(nq, nk, 64, seed=81)
    pre = oracle.prepass_head(q, k, v)
    o1 = oracle.attn_head(pre, causal=True)
    rng = np.random.default_rng(0)
    pre2 = {key: (val.copy() if isinstance(val, np.ndarray) else val) for key, val in pre.items()}
    pre2["k_hat"][cut:nk] = rng.integers(-127, 128, size=pre2["k_hat"][cut:nk].shape)
    pre2["dk_key"][cut:nk] = 0.5
    pre2["k_s"][cut:] = rng.standard_normal(pre2["k_s"][cut:].shape) * 10
    pre2["v_hat"][cut:] = rng.standard_normal(pre2["v_hat"][cut:].shape) * 100
    o2 = oracle.attn_head(pre2, causal=True)
    assert np.array_equal(o1[:cut], o2[:cut])
    assert np.all(np.any(o1[cut:] != o2[cut:], axis=1))


@pytest.mark.parametrize("gran", ["per_block", "per_threadgroup"])
def test_quality_against_full_precision_tiny_workload(gran):
    """The accuracy claim (cosine >= 0.995 against full-precision attention) on the tiny workload."""
    q, k, v = wl.generate(wl.TINY)
    qn, kn, vn = (x.double().numpy() for x in (q, k, v))
    o = oracle.sage_attention(qn, kn, vn, granularity=gran)
    ref = oracle.reference_attention(qn, kn, vn)
    cos = (o * ref).sum() / math.sqrt((o * o).sum() * (ref * ref).sum())
    assert cos >= 0.995


def test_empty_and_degenerate_heads():
    d = 64
    # a head with no keys: every row sees nothing, O = 0
    q = np.ones((5, d))
    k = np.zeros((0, d))
    v = np.zeros((0, d))
    pre = oracle.prepass_head(q, k, v)
    assert np.array_equal(oracle.attn_head(pre), np.zeros((5, d)))
    # causal with more queries than keys: the first n_q - n_kv rows see no key
    q, k, v = _rand_head(200, 100, d, seed=91)
    o = oracle.attn_head(oracle.prepass_head(q, k, v), causal=True)
    assert np.array_equal(o[:100], np.zeros((100, d)))
    assert np.all(np.abs(o[100:]).sum(1) > 0)
    # all-zero Q and K: scale 1, codes 0, uniform softmax -> O = mean of dequantized V
    q = np.zeros((130, d))
    k = np.zeros((140, d))
    v = np.tile(np.linspace(-1, 1, d), (140, 1))
    pre = oracle.prepass_head(q, k, v)
    assert np.all(pre["dq_row"] == 1.0) and np.all(pre["dk_key"] == 1.0)
    o = oracle.attn_head(pre)
    vdeq = (pre["v_hat"] * pre["dv"]).mean(0)
    assert np.max(np.abs(o - vdeq[None, :])) < 1e-12


# ---------------------------------------------------------------------------
# Grouped-query attention (H_kv key/value heads shared by H query heads)
# ---------------------------------------------------------------------------
def _gqa_inputs(B, H, H_kv, nq, nk, d, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, H, nq, d, generator=g).to(torch.bfloat16).double()
    k = (torch.randn(B, H_kv, nk, d, generator=g) + 3 * torch.randn(B, H_kv, 1, d, generator=g)).to(torch.bfloat16)
    v = torch.randn(B, H_kv, nk, d, generator=g).to(torch.bfloat16)
    return q, k.double(), v.double()


@pytest.mark.parametrize("causal", [False, True])
def test_gqa_unquantized_equals_torch_sdpa_enable_gqa(causal):
    """With the quantizers off, the oracle's grouped-query forward is torch's own
    grouped-query attention (scaled_dot_product_attention with enable_gqa), whose
    head grouping is the library's definition."""
    B, H, H_kv, nq, nk, d = 2, 6, 2, 150, 150, 64
    q, k, v = _gqa_inputs(B, H, H_kv, nq, nk, d, seed=5)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=causal, enable_gqa=True).numpy()
    o = oracle.sage_attention(q.numpy(), k.numpy(), v.numpy(), causal=causal, quant=(0, 0, 0))
    assert np.max(np.abs(o - ref)) < 1e-12
    r = oracle.reference_attention(q.numpy(), k.numpy(), v.numpy(), causal=causal)
    assert np.max(np.abs(r - ref)) < 1e-12


def test_gqa_equals_multi_head_on_repeated_kv_heads():
    """The quantized grouped-query forward equals the multi-head forward on K and V
    whose heads are repeated group-size times (torch.repeat_interleave), bit for bit:
    smoothing and delta_V depend on the key/value head alone."""
    B, H, H_kv, nq, nk, d = 1, 4, 2, 200, 260, 64
    q, k, v = _gqa_inputs(B, H, H_kv, nq, nk, d, seed=9)
    o = oracle.sage_attention(q.numpy(), k.numpy(), v.numpy(), causal=True)
    rep = H // H_kv
    o_mha = oracle.sage_attention(q.numpy(), k.repeat_interleave(rep, dim=1).numpy(),
                                  v.repeat_interleave(rep, dim=1).numpy(), causal=True)
    assert np.array_equal(o, o_mha)
    # tiling the heads instead (head h -> h % H_kv) is a different, wrong grouping
    o_tile = oracle.sage_attention(q.numpy(), k.repeat(1, rep, 1, 1).numpy(), v.repeat(1, rep, 1, 1).numpy(),
                                   causal=True)
    assert not np.array_equal(o[0, 1], o_tile[0, 1])


def test_gqa_bad_head_counts_rejected():
    q = np.zeros((1, 3, 4, 64))
    k = np.zeros((1, 2, 4, 64))
    with pytest.raises(ValueError):
        oracle.sage_attention(q, k, k)
    with pytest.raises(ValueError):
        oracle.reference_attention(q, k, k)


# ---------------------------------------------------------------------------
# Log-sum-exp of the rows
# ---------------------------------------------------------------------------
def _torch_lse(q, k, causal, scale):
    x = torch.from_numpy(q @ k.T) * scale
    if causal:
        nq, nk = q.shape[0], k.shape[0]
        vis = torch.arange(nk)[None, :] <= torch.arange(nq)[:, None] + (nk - nq)
        x = torch.where(vis, x, torch.tensor(-float("inf"), dtype=x.dtype))
    return torch.logsumexp(x, dim=1).numpy()


@pytest.mark.parametrize("smooth_q,smooth_k", [(True, True), (False, True), (True, False), (False, False)])
@pytest.mark.parametrize("causal,nq,nk", [(False, 200, 333), (True, 333, 200), (True, 256, 256)])
def test_lse_unquantized_equals_torch_logsumexp(smooth_q, smooth_k, causal, nq, nk):
    """With the quantizers off the method's row log-sum-exp, referred back to the
    unsmoothed logits, is torch.logsumexp of sm_scale * q . k (the K bias of these
    inputs shifts the smoothed logits by several units, so a missing correction fails)."""
    q, k, v = _rand_head(nq, nk, 64, seed=nq + nk, kbias=3.0, qbias=1.0)
    pre = oracle.prepass_head(q, k, v, quant=(0, 0, 0), smooth_q=smooth_q, smooth_k=smooth_k)
    lse = oracle.lse_head(pre, causal=causal)
    ref = _torch_lse(q, k, causal, 1 / 8)
    fin = np.isfinite(ref)
    assert np.array_equal(fin, np.isfinite(lse))
    assert np.max(np.abs(lse[fin] - ref[fin])) < 1e-11
    if causal and nq > nk:
        assert np.all(lse[:nq - nk] == -np.inf)


@pytest.mark.parametrize("gran,qbias", [("per_block", 0.0), ("per_threadgroup", 0.0), ("per_threadgroup", 20.0)])
def test_lse_quantized_within_logit_error_bound(gran, qbias):
    """Log-sum-exp is 1-Lipschitz in the largest logit change, and the row sum uses the
    unquantized P~, so each row's LSE lies within sm_scale times its largest INT8 score
    error bound, sum_c (dQ/2 |K_s| + dK/2 |Q_s| + dQ dK/4), of the exact value.  The
    bound holds whatever the Q channel offset, because the offset's part of the scores
    (qbar . K_s, the dS bias) is exact: the case with a large offset pins that."""
    nq, nk, d = 300, 400, 128
    q, k, v = _rand_head(nq, nk, d, seed=77, kbias=3.0, qbias=qbias)
    g_q, g_k = oracle.GRANULARITY[gran]
    pre = oracle.prepass_head(q, k, v, g_q=g_q, g_k=g_k)
    lse = oracle.lse_head(pre, causal=True)
    scale = 1 / math.sqrt(d)
    ref = _torch_lse(q, k, True, scale)
    qs = q - np.repeat(pre["qbar"].astype(np.float64), 128, axis=0)[:nq]
    ks = pre["k_s"]
    dq = pre["dq_row"][:nq].astype(np.float64)[:, None]
    dk = pre["dk_key"][:nk].astype(np.float64)[None, :]
    bound = (dq / 2) * np.abs(ks).sum(1)[None, :] + (dk / 2) * np.abs(qs).sum(1)[:, None] + d * dq * dk / 4
    vis = np.arange(nk)[None, :] <= np.arange(nq)[:, None] + (nk - nq)
    row_bound = scale * np.where(vis, bound, 0.0).max(1)
    err = np.abs(lse - ref)
    assert np.all(err <= row_bound + 1e-9)
    assert err.max() > 0   # the quantizers did act


# ---------------------------------------------------------------------------
# Packed variable-length batches
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [False, True])
def test_varlen_unquantized_equals_block_diagonal_masked_sdpa(causal):
    """With the quantizers off the packed-batch forward is attention over the whole
    packed token axis under a block-diagonal mask (each token sees only its own
    sequence; causal bottom-right aligned inside each block), computed by torch's
    scaled_dot_product_attention with an explicit boolean mask."""
    g = torch.Generator().manual_seed(12)
    lq, lk = [70, 1, 200, 129], [90, 5, 200, 60]
    cu_q, cu_kv = np.concatenate([[0], np.cumsum(lq)]), np.concatenate([[0], np.cumsum(lk)])
    H, H_kv, d = 4, 2, 64
    q = torch.randn(cu_q[-1], H, d, generator=g, dtype=torch.float64)
    k = torch.randn(cu_kv[-1], H_kv, d, generator=g, dtype=torch.float64) + 2.0
    v = torch.randn(cu_kv[-1], H_kv, d, generator=g, dtype=torch.float64)
    o = oracle.sage_attention_varlen(q.numpy(), k.numpy(), v.numpy(), cu_q, cu_kv, causal=causal, quant=(0, 0, 0))
    seq_q = np.repeat(np.arange(len(lq)), lq)
    seq_k = np.repeat(np.arange(len(lk)), lk)
    pos_q = np.arange(cu_q[-1]) - cu_q[seq_q]
    pos_k = np.arange(cu_kv[-1]) - cu_kv[seq_k]
    mask = seq_q[:, None] == seq_k[None, :]
    if causal:
        off = (np.asarray(lk) - np.asarray(lq))[seq_q]
        mask &= pos_k[None, :] <= pos_q[:, None] + off[:, None]
    m = torch.from_numpy(mask)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.permute(1, 0, 2)[None], k.permute(1, 0, 2)[None], v.permute(1, 0, 2)[None], attn_mask=m,
        enable_gqa=True)[0].permute(1, 0, 2).numpy()
    seen = mask.any(1)   # rows with no visible key: SDPA gives NaN, the method 0
    assert np.max(np.abs(o[seen] - ref[seen])) < 1e-12
    assert np.all(o[~seen] == 0)


# ---------------------------------------------------------------------------
# FP16 P / V mode ("qk_int8_pv_fp16")
# ---------------------------------------------------------------------------
def test_f16_codec_matches_numpy():
    """The oracle's fp16 rounding against numpy's float32 -> float16 conversion (IEEE,
    ties to even) on random values spanning the subnormals, the normals, the largest
    finite value and overflow."""
    rng = np.random.default_rng(3)
    x = np.concatenate([
        rng.standard_normal(4000).astype(np.float32) * np.float32(2.0) ** rng.integers(-30, 17, 4000),
        np.float32([0.0, -0.0, 65504.0, 65519.0, 65520.0, -65520.0, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26,
                    2.0 ** -14, 1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11])]).astype(np.float32)
    got = oracle.f16_round(x)
    with np.errstate(over="ignore"):   # 65520 and beyond overflow to inf, as IEEE rounding does
        ref = x.astype(np.float16).astype(np.float64)
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("causal", [False, True])
def test_pv_fp16_with_exact_qk_equals_attention_with_fp16_operands(causal):
    """With exact QK^T, one key tile (so the online softmax is the two-pass one) and
    FP16 P / V, the oracle equals softmax attention whose P~ = exp(x - m) and V are
    rounded to fp16 (numpy's float16) before the PV product, divided by the unrounded
    row sum."""
    nq, nk, d = 200, 128, 64
    q, k, v = _rand_head(nq, nk, d, seed=404, kbias=2.0, outliers=False)
    pre = oracle.prepass_head(q, k, v, quant=(0, 2, 2))
    o = oracle.attn_head(pre, causal=causal)
    x = (q @ k.T) / 8.0
    if causal:
        x = np.where(np.arange(nk)[None, :] <= np.arange(nq)[:, None] + (nk - nq), x, -np.inf)
    seen = np.isfinite(x).any(1)
    m = np.where(seen, x.max(1), 0.0)[:, None]
    p = np.exp(x - m)
    p16 = p.astype(np.float32).astype(np.float16).astype(np.float64)
    v16 = v.astype(np.float32).astype(np.float16).astype(np.float64)
    ref = np.zeros_like(o)
    ref[seen] = (p16[seen] @ v16) / p[seen].sum(1, keepdims=True)
    assert np.max(np.abs(o - ref)) < 1e-12
    assert np.all(pre["dv"] == 1.0)
    assert np.any(p16 != p)   # the rounding acted


def test_pv_fp16_more_accurate_than_fp8():
    """The FP16 P / V mode is closer to full-precision attention than FP8 P / V."""
    q, k, v = wl.generate(wl.TINY)
    qn, kn, vn = (x.double().numpy() for x in (q, k, v))
    ref = oracle.reference_attention(qn, kn, vn)
    o8 = oracle.sage_attention(qn, kn, vn, quant=oracle.PV_FP8)
    o16 = oracle.sage_attention(qn, kn, vn, quant=oracle.PV_FP16)
    e8, e16 = np.abs(o8 - ref).max(), np.abs(o16 - ref).max()
    assert e16 < e8


# ---------------------------------------------------------------------------
# FP4 (E2M1) Q / K with two-level scales
# ---------------------------------------------------------------------------
def _e2m1_value(code):
    """E2M1 from its definition: sign bit 3, exponent bits 2-1 (bias 1), mantissa bit 0."""
    s, e, m = (code >> 3) & 1, (code >> 1) & 3, code & 1
    v = m * 0.5 if e == 0 else 2.0 ** (e - 1) * (1 + m / 2)
    return -v if s else v


def test_e2m1_codec_against_definition_and_brute_force():
    assert [oracle.e2m1_decode(c) for c in range(16)] == [_e2m1_value(c) for c in range(16)]
    finite = sorted({_e2m1_value(c) for c in range(16)})
    rng = np.random.default_rng(8)
    mids = [(a + b) / 2 for a, b in zip(finite, finite[1:])]
    xs = np.concatenate([rng.uniform(-7, 7, 3000), mids, [0.0, 6.0, -6.0, 6.5, -100.0, 5.999]]).astype(np.float32)
    codes = oracle.e2m1_encode(xs)
    for x, c in zip(xs, codes):
        if abs(x) >= 6:
            assert oracle.e2m1_decode(c) == np.sign(x) * 6
            continue
        dist = [abs(float(x) - f) for f in finite]
        best = min(dist)
        cands = [finite[i] for i, dd in enumerate(dist) if dd == best]
        if len(cands) == 1:
            assert oracle.e2m1_decode(c) == cands[0]
        else:  # a tie goes to the value with an even mantissa bit
            even = [f for f in cands if int(oracle.e2m1_encode(np.float32([f]))[0]) & 1 == 0]
            assert oracle.e2m1_decode(c) == even[0]


def test_fp4_block_scales_reconstruct_within_half_a_code_step():
    """x ~ g * sf * code per 16-channel block: the reconstruction error of every
    element is at most half the E2M1 spacing at its code (saturated elements excepted),
    every block's largest element codes to 4 or 6, and q_hat is sf * code."""
    q, k, v = _rand_head(200, 300, 128, seed=55, kbias=3.0, qbias=1.0)
    pre = oracle.prepass_head(q, k, v, quant=oracle.QK_FP4_PV_FP8)
    qs = (q - np.repeat(pre["qbar"].astype(np.float64), 128, axis=0)[:200]).astype(np.float32)
    g = pre["dq_row"][:200].astype(np.float64)
    sf = np.array([[oracle.e4m3_decode(c) for c in row] for row in pre["q_sf"][:200]])
    codes = pre["q_code"][:200].astype(np.uint8)
    a = oracle.e2m1_decode(codes)
    delta = np.repeat(sf, 16, axis=1) * g[:, None]
    assert np.array_equal(pre["q_hat"][:200], np.repeat(sf, 16, axis=1) * a)
    spacing = np.where(np.abs(a) < 2, 0.5, np.where(np.abs(a) < 4, 1.0, 2.0))
    err = np.abs(qs - delta * a)
    ok = (err <= delta * spacing / 2 * (1 + 1e-6)) | (np.abs(a) == 6)
    assert ok.all()
    blk_max = np.abs(a).reshape(200, 8, 16).max(2)
    xs_max = np.abs(qs).reshape(200, 8, 16).max(2)
    assert np.all((blk_max >= 4) | (xs_max == 0))


def test_fp4_tile_scale_puts_the_largest_block_at_the_top_of_e4m3():
    """The per-tile fp32 scale g exists to keep the E4M3 block scales in range while
    using all of it (the microscaling form of 4-bit operands, "SageAttention3:
    Microscaling FP4 Attention" in the notes' related-papers table; the 4-bit QK of the
    SageAttention2 abstract): in every 128-row tile with a nonzero entry, the 16-channel
    block that holds the tile's largest magnitude gets the largest finite E4M3 scale,
    448 (code 0x7E), and its largest element codes to E2M1 6, so that g = amax / 2688
    follows from 6 * 448 * g = amax.  Checked on Q (three tiles, one ragged) and K."""
    q, k, v = _rand_head(300, 270, 128, seed=57, kbias=3.0, qbias=1.0)
    pre = oracle.prepass_head(q, k, v, quant=oracle.QK_FP4_PV_FP8)
    for x, bar, sf_all, code_all, n in (
            (q, np.repeat(pre["qbar"].astype(np.float64), 128, axis=0), pre["q_sf"], pre["q_code"], 300),
            (k, pre["kbar"].astype(np.float64)[None, :], pre["k_sf"], pre["k_code"], 270)):
        xs = np.zeros((-(-n // 128) * 128, 128), np.float32)
        xs[:n] = (x - bar[:n] if bar.shape[0] > 1 else x - bar).astype(np.float32)
        for t in range(xs.shape[0] // 128):
            tile = np.abs(xs[128 * t:128 * (t + 1)])
            r, c = np.unravel_index(np.argmax(tile), tile.shape)
            assert tile[r, c] > 0
            assert sf_all[128 * t + r, c // 16] == 0x7E
            assert oracle.e2m1_decode(code_all[128 * t + r, c]) in (6.0, -6.0)
            # no block scale exceeds the top one
            assert np.all(np.array([[oracle.e4m3_decode(s) for s in row]
                                    for row in sf_all[128 * t:128 * (t + 1)]]) <= 448.0)


def test_fp4_block_scale_that_underflows_e4m3_is_the_smallest_subnormal():
    """A 16-channel block far below the tile maximum has amax / g / 6 below half of
    E4M3's smallest subnormal 2^-9, which rounds to 0; a zero scale would divide by 0,
    so the block takes the smallest positive scale 2^-9 (code 0x01) and its elements
    code to 0.  Crafted tile: one entry 1000, one block with entries of 1e-6, the rest 0
    (an all-zero block keeps the scale 1.0, code 0x38)."""
    nq, d = 128, 64
    q = np.zeros((nq, d))
    q[3, 5] = 1000.0
    q[70, 16:32] = 1e-6
    k = np.eye(128, d)
    v = np.ones((128, d))
    pre = oracle.prepass_head(q, k, v, quant=oracle.QK_FP4_PV_FP8, smooth_q=False)
    g = 1000.0 / 2688.0
    assert (1e-6 / g) / 6 < 2.0 ** -10          # rounds to E4M3 zero
    assert pre["q_sf"][70, 1] == 0x01
    assert oracle.e4m3_decode(0x01) == 2.0 ** -9
    assert np.all(oracle.e2m1_decode(pre["q_code"][70, 16:32]) == 0.0)
    assert pre["q_sf"][3, 0] == 0x7E
    assert pre["q_sf"][70, 0] == 0x38 and pre["q_sf"][0, 2] == 0x38


def test_fp4_scores_equal_attention_on_dequantized_q_k():
    """With FP4 Q / K and exact P / V, the oracle is textbook attention on the
    dequantized smoothed operands plus the Q-smoothing bias (numpy, from the pre-pass
    codes and scales)."""
    nq, nk, d = 150, 260, 64
    q, k, v = _rand_head(nq, nk, d, seed=66, kbias=3.0, qbias=1.0)
    pre = oracle.prepass_head(q, k, v, quant=(2, 0, 0))
    o = oracle.attn_head(pre, causal=True)
    qh = pre["q_hat"][:nq] * pre["dq_row"][:nq, None].astype(np.float64)
    kh = pre["k_hat"][:nk] * pre["dk_key"][:nk, None].astype(np.float64)
    tq = -(-nq // 128)
    ds = np.stack([oracle.delta_s(pre, t) for t in range(tq)])
    s = qh @ kh.T + ds[np.arange(nq) // 128]
    ref = _textbook_from_scores(s / 8.0, v, causal=True)
    assert np.max(np.abs(o - ref)) < 1e-12


def _textbook_from_scores(x, v, causal):
    nq, nk = x.shape
    if causal:
        x = np.where(np.arange(nk)[None, :] <= np.arange(nq)[:, None] + (nk - nq), x, -np.inf)
    m = x.max(1, keepdims=True)
    p = np.exp(x - m)
    return (p @ v) / p.sum(1, keepdims=True)


def test_fp4_qk_accuracy_and_smoothing():
    """FP4 Q / K is lossier than INT8 but close to full precision on the tiny workload
    (cosine >= 0.985 against 0.999 for INT8), and without K smoothing a large K bias
    ruins it (inputs with a per-channel K bias of std 8)."""
    q, k, v = wl.generate(wl.TINY)
    qn, kn, vn = (x.double().numpy() for x in (q, k, v))
    ref = oracle.reference_attention(qn, kn, vn)
    o4 = oracle.sage_attention(qn, kn, vn, quant=oracle.QK_FP4_PV_FP8)
    o8 = oracle.sage_attention(qn, kn, vn, quant=oracle.PV_FP8)
    assert 0.985 <= cos_np(o4, ref) < cos_np(o8, ref)
    qb, kb, vb = _rand_head(256, 256, 64, seed=77, kbias=8.0)
    r = oracle.reference_attention(qb[None, None], kb[None, None], vb[None, None])[0, 0]
    on = oracle.attn_head(oracle.prepass_head(qb, kb, vb, quant=oracle.QK_FP4_PV_FP8, smooth_k=False))
    os_ = oracle.attn_head(oracle.prepass_head(qb, kb, vb, quant=oracle.QK_FP4_PV_FP8))
    assert cos_np(os_, r) > 0.9 > 0.7 > cos_np(on, r)


def cos_np(a, b):
    a, b = np.ravel(a), np.ravel(b)
    return float(a @ b / math.sqrt((a @ a) * (b @ b)))


def test_q_block_means_of_ragged_blocks():
    """q̄ of each 128-row block is the fp64 mean of its valid rows (numpy), rounded once
    to fp32: the ragged last block averages its 72 rows, not 128."""
    q, k, v = _rand_head(200, 130, 64, seed=88, qbias=2.0)
    pre = oracle.prepass_head(q, k, v)
    for t, (r0, r1) in enumerate(((0, 128), (128, 200))):
        assert np.array_equal(pre["qbar"][t], q[r0:r1].mean(axis=0).astype(np.float32))
    assert np.array_equal(pre["kbar"], k.mean(axis=0).astype(np.float32))
