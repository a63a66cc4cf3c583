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


def _atoms(sf, n_pad, d):
    """[n_pad, d/16] E4M3 scale codes -> [n_pad/128, d/64, 512] atoms (row m, block b at byte
    16 (m mod 32) + 4 (m / 32) + (b mod 4) of atom b / 4)."""
    out = np.zeros((n_pad // 128, d // 64, 512), np.uint8)
    m = np.arange(128)
    for t in range(n_pad // 128):
        for b in range(d // 16):
            out[t, b // 4, 16 * (m % 32) + 4 * (m // 32) + (b % 4)] = sf[t * 128 + m, b]
    return out


@pytest.mark.parametrize("d,nq,nk,recipe", [(64, 300, 333, "llm"), (128, 200, 129, "image_dit"),
                                            (64, 128, 1000, "video_dit")])
def test_fp4_prepass_bit_exact(d, nq, nk, recipe):
    """sage_quant_qk in the 4-bit mode: Q / K codes, the scale atoms and the per-tile
    scales (in delta_Q's and delta_K's places) equal the oracle's FP4 mode bit for bit,
    and so do qbar, kbar and the row shift of the LSE."""
    w = wl.custom("fp4pre", 1, 2, nq, nk, d, False, recipe=recipe, seed=8800 + d + nq)
    q, k, v = wl.generate(w)
    mode = sage.QuantMode.make("fp4")
    ws = sage.quant_qk(q.cuda(), k.cuda(), mode=mode)
    torch.cuda.synchronize()
    nq_pad, nk_pad = -(-nq // 128) * 128, -(-nk // 128) * 128
    for h in range(w.H):
        pre = oracle.prepass_head(q[0, h].double().numpy(), k[0, h].double().numpy(), v[0, h].double().numpy(),
                                  quant=oracle.QK_FP4_PV_FP8)
        assert np.array_equal(ws.view("q8")[h].cpu().numpy(), _pack(pre["q_code"])), "Q codes"
        assert np.array_equal(ws.view("k8")[h].cpu().numpy(), _pack(pre["k_code"])), "K codes"
        assert np.array_equal(ws.view("sfq")[h].cpu().numpy(), _atoms(pre["q_sf"], nq_pad, d)), "Q scale atoms"
        assert np.array_equal(ws.view("sfk")[h].cpu().numpy(), _atoms(pre["k_sf"], nk_pad, d)), "K scale atoms"
        assert np.array_equal(ws.view("dq")[h].cpu().numpy(), pre["dq_row"]), "Q tile scales"
        assert np.array_equal(ws.view("dk")[h].cpu().numpy(), pre["dk_key"][::16]), "K tile scales"
        assert np.array_equal(ws.view("qbar")[h].cpu().numpy(), pre["qbar"])
        assert np.array_equal(ws.view("kbar")[h].cpu().numpy(), pre["kbar"])


@pytest.mark.parametrize("B,H,Hk,nq,nk,causal,layout,dtype,recipe", [
    (1, 2, 2, 256, 256, False, "HND", torch.float16, "video_dit"),   # the tiny workload's shape
    (2, 3, 3, 300, 333, True, "HND", torch.bfloat16, "llm"),         # ragged tails, causal, N_q != N_kv
    (1, 4, 2, 513, 700, False, "NHD", torch.bfloat16, "llm"),        # grouped-query heads, token-major
])
def test_fp4_attention_matches_oracle(B, H, Hk, nq, nk, causal, layout, dtype, recipe):
    """O of the 4-bit mode (QK^T on kind::mxf4nvf4, d = 64) against the oracle's FP4 Q / K
    mode within the O tolerance, and its LSE within 1e-3.  (bf16 output is compared on
    V ~ N(0, 1): with the video recipe's channel scales up to 10, bf16 rounding of O alone
    reaches the 1e-2 bound against the unrounded fp64 oracle.)"""
    from helpers import assert_close_to_oracle, to_np64
    w = wl.custom("fp4attn", B, H, nq, nk, 64, causal, dtype=dtype, recipe=recipe, seed=8900 + nq, H_kv=Hk)
    q, k, v = wl.generate(w)
    if layout == "NHD":
        q, k, v = (x.transpose(1, 2).contiguous() for x in (q, k, v))
    o, lse = sage.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, layout=layout, granularity="fp4",
                           return_lse=True)
    o = o.cpu()
    if layout == "NHD":
        o, q, k, v = (x.transpose(1, 2) for x in (o, q, k, v))
    lse = lse.cpu().double().numpy()
    g = H // Hk
    for b in range(B):
        for h in range(H):
            pre = oracle.prepass_head(to_np64(q[b, h]), to_np64(k[b, h // g]), to_np64(v[b, h // g]),
                                      quant=oracle.QK_FP4_PV_FP8)
            oo = oracle.attn_head(pre, causal=causal)
            assert_close_to_oracle(to_np64(o[b, h]), oo, "fp4 (%d,%d)" % (b, h))
            ll = oracle.lse_head(pre, causal=causal)
            assert np.max(np.abs(lse[b, h] - ll)) <= 1e-3, "fp4 LSE (%d,%d)" % (b, h)


def test_fp4_attention_varlen_matches_dense_calls():
    """Packed sequences in the 4-bit mode equal per-sequence dense calls bit for bit."""
    lens = [(200, 300), (0, 17), (129, 129), (64, 500)]
    H, Hk, d = 4, 2, 64
    g = torch.Generator().manual_seed(8950)
    qs = [torch.randn(nq, H, d, generator=g).bfloat16() for nq, _ in lens]
    ks = [(torch.randn(nk, Hk, d, generator=g) + 3 * torch.randn(1, Hk, d, generator=g)).bfloat16() for _, nk in lens]
    vs = [torch.randn(nk, Hk, d, generator=g).bfloat16() for _, nk in lens]
    cu_q = torch.tensor([0] + list(np.cumsum([a for a, _ in lens])), dtype=torch.int32)
    cu_k = torch.tensor([0] + list(np.cumsum([b for _, b in lens])), dtype=torch.int32)
    o = sage.attn_fwd_varlen(torch.cat(qs).cuda(), torch.cat(ks).cuda(), torch.cat(vs).cuda(), cu_q.cuda(),
                             cu_k.cuda(), causal=True, granularity="fp4").cpu()
    for i, (nq, nk) in enumerate(lens):
        if nq == 0:
            continue
        ref = sage.attn_fwd(qs[i][None].cuda(), ks[i][None].cuda(), vs[i][None].cuda(), causal=True, layout="NHD",
                            granularity="fp4").cpu()[0]
        assert torch.equal(o[int(cu_q[i]):int(cu_q[i + 1])], ref), "sequence %d" % i


def test_fp4_attention_refuses_d128():
    q = torch.zeros((1, 1, 128, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sage.SageError) as e:
        sage.attn_fwd(q, q, q, granularity="fp4")
    assert e.value.code == sage.SAGE_ERR_UNSUPPORTED
