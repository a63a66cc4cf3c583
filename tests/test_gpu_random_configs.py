"""Seeded random configurations through the whole forward, against the oracle.

Each case draws its sizes and options from one seeded generator: batch and heads
(grouped-query included), ragged query and key lengths on both sides of the 128-row
tile, d, causal or not, dtype, layout, Q / K granularity, FP8 or FP16 P / V, Q
smoothing on or off, an sm_scale, and a Q channel offset (so that the Q smoothing bias
dS is not near zero).  The output of every head is compared with the oracle run on that
head at the usual tolerance, and so is the LSE.  Half of the cases run the path that
quantizes Q inside the attention kernel.
"""
import numpy as np
import pytest
import torch

import oracle
import quantized_attention_fine_b200 as sage

from helpers import GRAN_OF, assert_close_to_oracle, to_np64

pytestmark = pytest.mark.gpu

N_CASES = 16


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from quantized_attention_fine_b200 import _build
    _build.build()
    sage.load_library()


def _draw(seed):
    r = np.random.default_rng(5000 + seed)
    H_kv = int(r.choice([1, 2, 3]))
    cfg = dict(
        B=int(r.integers(1, 3)), H_kv=H_kv, H=H_kv * int(r.choice([1, 2, 4])),
        nq=int(r.choice([1, 77, 128, 129, 255, 300, 513])), nk=int(r.choice([1, 100, 128, 200, 384, 641])),
        d=int(r.choice([64, 128])), causal=bool(r.integers(0, 2)),
        dtype=[torch.float16, torch.bfloat16][int(r.integers(0, 2))], layout=["HND", "NHD"][int(r.integers(0, 2))],
        gran=["per_threadgroup", "per_warp", "per_block"][int(r.integers(0, 3))],
        pv=["fp8", "fp16"][int(r.integers(0, 2))] if r.random() < 0.3 else "fp8",
        smooth_q=bool(r.random() < 0.8), sm_scale=float(r.choice([0.0, 0.05, 0.2])),
        q_bias=float(r.choice([0.0, 2.0, 6.0])), fuse_q=bool(seed % 2),
    )
    g = torch.Generator().manual_seed(6000 + seed)
    B, H, Hk, nq, nk, d = cfg["B"], cfg["H"], cfg["H_kv"], cfg["nq"], cfg["nk"], cfg["d"]
    q = torch.randn((B, H, nq, d), generator=g) + cfg["q_bias"] * torch.randn((B, H, 1, d), generator=g)
    k = torch.randn((B, Hk, nk, d), generator=g) + 3.0 * torch.randn((B, Hk, 1, d), generator=g)
    v = torch.randn((B, Hk, nk, d), generator=g)
    q, k, v = (x.to(cfg["dtype"]) for x in (q, k, v))
    return cfg, q, k, v


@pytest.mark.parametrize("seed", range(N_CASES))
def test_random_configuration(seed):
    cfg, q, k, v = _draw(seed)
    to_dev = (lambda x: x.cuda()) if cfg["layout"] == "HND" else (lambda x: x.permute(0, 2, 1, 3).contiguous().cuda())
    o, lse = sage.attn_fwd(to_dev(q), to_dev(k), to_dev(v), causal=cfg["causal"], sm_scale=cfg["sm_scale"] or None,
                           layout=cfg["layout"], granularity=cfg["gran"], smooth_q=cfg["smooth_q"], pv=cfg["pv"],
                           return_lse=True, fuse_q=cfg["fuse_q"])
    torch.cuda.synchronize()
    o = o.cpu()
    if cfg["layout"] == "NHD":
        o = o.permute(0, 2, 1, 3)
    lse = lse.cpu().double().numpy()
    g_q, g_k = GRAN_OF[cfg["gran"]]
    quant = oracle.PV_FP16 if cfg["pv"] == "fp16" else (1, 1, 1)
    group = cfg["H"] // cfg["H_kv"]
    what = "seed %d %s" % (seed, {k_: (str(v_) if k_ == "dtype" else v_) for k_, v_ in cfg.items()})
    for b in range(cfg["B"]):
        for h in range(cfg["H"]):
            pre = oracle.prepass_head(to_np64(q[b, h]), to_np64(k[b, h // group]), to_np64(v[b, h // group]), g_q=g_q,
                                      g_k=g_k, smooth_q=cfg["smooth_q"], quant=quant)
            oo = oracle.attn_head(pre, causal=cfg["causal"], sm_scale=cfg["sm_scale"] or None)
            assert_close_to_oracle(to_np64(o[b, h]), oo, what + " head (%d,%d)" % (b, h))
            ll = oracle.lse_head(pre, causal=cfg["causal"], sm_scale=cfg["sm_scale"] or None)
            fin = np.isfinite(ll)
            got = lse[b, h, :cfg["nq"]]
            assert np.array_equal(np.isfinite(got), fin), what + ": LSE finite pattern"
            if fin.any():
                assert np.max(np.abs(got[fin] - ll[fin])) <= 1e-3, what + ": LSE"


N_VARLEN = 8


@pytest.mark.parametrize("seed", range(N_VARLEN))
def test_random_packed_batch(seed):
    """Packed variable-length batches (empty sequences, one-token sequences, q shorter or
    longer than kv), drawn like the dense cases, against the oracle's packed forward."""
    r = np.random.default_rng(7000 + seed)
    nb = int(r.integers(1, 5))
    H_kv = int(r.choice([1, 2]))
    H = H_kv * int(r.choice([1, 2, 3]))
    d = int(r.choice([64, 128]))
    dtype = [torch.float16, torch.bfloat16][int(r.integers(0, 2))]
    causal = bool(r.integers(0, 2))
    gran = ["per_threadgroup", "per_warp", "per_block"][int(r.integers(0, 3))]
    pv = "fp16" if r.random() < 0.25 else "fp8"
    fuse_q = bool(seed % 2)
    lq = [int(x) for x in r.choice([0, 1, 90, 128, 200, 333], size=nb)]
    lk = [int(x) for x in r.choice([1, 64, 128, 250, 400], size=nb)]
    g = torch.Generator().manual_seed(8000 + seed)
    q = torch.randn(sum(lq), H, d, generator=g) + 3.0 * torch.randn(1, H, d, generator=g)
    k = torch.randn(sum(lk), H_kv, d, generator=g) + 3.0 * torch.randn(1, H_kv, d, generator=g)
    v = torch.randn(sum(lk), H_kv, d, generator=g)
    q, k, v = (x.to(dtype) for x in (q, k, v))
    cu_q = np.concatenate([[0], np.cumsum(lq)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lk)]).astype(np.int32)
    o, lse = sage.attn_fwd_varlen(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(cu_q).cuda(),
                                  torch.from_numpy(cu_k).cuda(), causal=causal, granularity=gran, pv=pv,
                                  return_lse=True, fuse_q=fuse_q)
    torch.cuda.synchronize()
    o = o.cpu()
    lse = lse.cpu().double().numpy()
    oo, ll = oracle.sage_attention_varlen(to_np64(q), to_np64(k), to_np64(v), cu_q, cu_k, causal=causal,
                                          return_lse=True, granularity=gran,
                                          quant=oracle.PV_FP16 if pv == "fp16" else (1, 1, 1))
    what = "seed %d: lq %s lk %s H %d/%d d %d causal %s %s pv %s fuse_q %s" % (seed, lq, lk, H, H_kv, d, causal,
                                                                             gran, pv, fuse_q)
    for b in range(nb):
        q0, q1 = int(cu_q[b]), int(cu_q[b + 1])
        for h in range(H):
            if q1 > q0:
                assert_close_to_oracle(to_np64(o[q0:q1, h]), oo[q0:q1, h], what + " seq %d head %d" % (b, h))
                ref = ll[q0:q1, h]
                got = lse[b, h, :q1 - q0]
                fin = np.isfinite(ref)
                assert np.array_equal(np.isfinite(got), fin), what + ": LSE finite pattern"
                if fin.any():
                    assert np.max(np.abs(got[fin] - ref[fin])) <= 1e-3, what + ": LSE"
