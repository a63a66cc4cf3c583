"""Packed variable-length batches on the GPU (sage_attn_fwd_varlen, through the C ABI).

Each sequence is checked against the oracle run on that sequence alone, and the packed
call against per-sequence dense calls on the same tokens, which make the same integer
decisions and so give identical bits.
"""
import numpy as np
import pytest
import torch

import oracle
import quantized_attention_fine_b200 as sage

from helpers import O_COS_FULL, assert_close_to_oracle, cos, to_np64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from quantized_attention_fine_b200 import _build
    _build.build()
    sage.load_library()


def _packed(lq, lk, H, H_kv, d, seed, dtype=torch.bfloat16, kbias=3.0):
    g = torch.Generator().manual_seed(seed)
    tq, tk = int(sum(lq)), int(sum(lk))
    q = torch.randn(tq, H, d, generator=g)
    mask = torch.rand(tq, H, d, generator=g) < 0.01
    q = torch.where(mask, q * 20, q)
    k = torch.randn(tk, H_kv, d, generator=g) + kbias * torch.randn(1, H_kv, d, generator=g)
    v = torch.randn(tk, H_kv, d, generator=g)
    cu_q = np.concatenate([[0], np.cumsum(lq)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lk)]).astype(np.int32)
    return q.to(dtype), k.to(dtype), v.to(dtype), cu_q, cu_k


CASES = [
    # name, q lengths, kv lengths, H, H_kv, d, causal, dtype
    ("mixed_d128", [300, 1, 128, 517, 64], [300, 1, 128, 517, 64], 2, 2, 128, False, torch.bfloat16),
    ("mixed_causal_d64", [250, 700, 33, 129], [250, 700, 33, 129], 4, 4, 64, True, torch.bfloat16),
    ("q_ne_kv_causal_gqa", [100, 300, 257], [300, 100, 257], 8, 2, 128, True, torch.float16),
    ("empty_sequences", [0, 200, 130, 0], [50, 0, 130, 90], 2, 1, 64, False, torch.bfloat16),
]


@pytest.mark.parametrize("name,lq,lk,H,Hk,d,causal,dtype", CASES, ids=[c[0] for c in CASES])
def test_varlen_matches_oracle_per_sequence(name, lq, lk, H, Hk, d, causal, dtype):
    q, k, v, cu_q, cu_k = _packed(lq, lk, H, Hk, d, seed=9000 + len(name), dtype=dtype)
    o, lse = sage.attn_fwd_varlen(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(cu_q).cuda(),
                                  torch.from_numpy(cu_k).cuda(), causal=causal, return_lse=True)
    o = to_np64(o)
    lse = to_np64(lse)
    oo, ll = oracle.sage_attention_varlen(to_np64(q), to_np64(k), to_np64(v), cu_q, cu_k, causal=causal,
                                          return_lse=True)
    for b in range(len(lq)):
        q0, q1 = cu_q[b], cu_q[b + 1]
        if q1 == q0:
            continue
        for h in range(H):
            assert_close_to_oracle(o[q0:q1, h], oo[q0:q1, h], "%s seq %d head %d" % (name, b, h))
            got, ref = lse[b, h, :q1 - q0], ll[q0:q1, h]
            fin = np.isfinite(ref)
            assert np.array_equal(np.isfinite(got), fin)
            if fin.any():
                assert np.max(np.abs(got[fin] - ref[fin])) <= 1e-3
    ref_full = np.zeros_like(oo)
    for b in range(len(lq)):
        q0, q1, k0, k1 = cu_q[b], cu_q[b + 1], cu_k[b], cu_k[b + 1]
        if q1 > q0 and k1 > k0:
            for h in range(H):
                ref_full[q0:q1, h] = oracle.reference_attention(
                    to_np64(q[q0:q1, h])[None, None], to_np64(k[k0:k1, h // (H // Hk)])[None, None],
                    to_np64(v[k0:k1, h // (H // Hk)])[None, None], causal=causal)[0, 0]
    assert cos(o, ref_full) >= O_COS_FULL


def test_varlen_equals_dense_calls_bit_exact():
    lq = [300, 129, 520, 1]
    lk = [400, 129, 520, 77]
    H, Hk, d = 4, 2, 128
    q, k, v, cu_q, cu_k = (x for x in _packed(lq, lk, H, Hk, d, seed=9100))
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o, lse = sage.attn_fwd_varlen(qd, kd, vd, torch.from_numpy(cu_q).cuda(), torch.from_numpy(cu_k).cuda(),
                                  causal=True, return_lse=True)
    o, lse = o.clone(), lse.clone()
    for b in range(len(lq)):
        q0, q1, k0, k1 = cu_q[b], cu_q[b + 1], cu_k[b], cu_k[b + 1]
        ob, lb = sage.attn_fwd(qd[q0:q1][None].contiguous(), kd[k0:k1][None].contiguous(),
                               vd[k0:k1][None].contiguous(), causal=True, layout="NHD", return_lse=True)
        torch.cuda.synchronize()
        assert torch.equal(o[q0:q1], ob[0]), "sequence %d" % b
        assert torch.equal(lse[b, :, :q1 - q0], lb[0]), "LSE of sequence %d" % b


def test_varlen_uncovered_tokens_untouched_and_long_batch_deterministic():
    """Offsets that end before total_q leave the remaining output tokens as they were;
    a packed batch of long sequences (all SMs busy) is deterministic."""
    lq = [4096, 1000, 8192, 300, 2048]
    H, Hk, d = 8, 2, 128
    q, k, v, cu_q, cu_k = _packed(lq, lq, H, Hk, d, seed=9200)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    extra = 64   # tokens past the last sequence
    qx = torch.cat([qd, torch.zeros(extra, H, d, dtype=qd.dtype, device="cuda")])
    cq, ck = torch.from_numpy(cu_q).cuda(), torch.from_numpy(cu_k).cuda()
    outs = []
    for _ in range(3):
        o = torch.full_like(qx, 5.0)
        sage.attn_fwd_varlen(qx, kd, vd, cq, ck, causal=True, out=o)
        outs.append(o)
    torch.cuda.synchronize()
    for o in outs:
        assert torch.all(o[-extra:] == 5.0)
        assert torch.equal(o, outs[0])
    # sampled oracle check: the last Q block of two sequences, every head
    o = to_np64(outs[0])
    for b in (0, 2):
        q0, n = cu_q[b], lq[b]
        for h in (0, H - 1):
            pre = oracle.prepass_head(to_np64(q[q0:q0 + n, h]), to_np64(k[q0:q0 + n, h // (H // Hk)]),
                                      to_np64(v[q0:q0 + n, h // (H // Hk)]))
            tq = -(-n // 128)
            oo = oracle.attn_head(pre, causal=True, qblocks=[tq - 1])
            rows = np.arange((tq - 1) * 128, n)
            assert_close_to_oracle(o[q0 + rows, h], oo[rows], "seq %d head %d" % (b, h))


def test_varlen_fp16_inputs_d64():
    lq = [129, 1, 640, 77]
    lk = [300, 64, 640, 77]
    H, Hk, d = 4, 4, 64
    q, k, v, cu_q, cu_k = _packed(lq, lk, H, Hk, d, seed=9960, dtype=torch.float16)
    o = sage.attn_fwd_varlen(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(cu_q).cuda(),
                             torch.from_numpy(cu_k).cuda(), causal=True)
    assert o.dtype == torch.float16
    o = to_np64(o)
    oo = oracle.sage_attention_varlen(to_np64(q), to_np64(k), to_np64(v), cu_q, cu_k, causal=True)
    for b in range(len(lq)):
        q0, q1 = cu_q[b], cu_q[b + 1]
        for h in range(H):
            assert_close_to_oracle(o[q0:q1, h], oo[q0:q1, h], "seq %d head %d" % (b, h))
