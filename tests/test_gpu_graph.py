"""The whole forward captured in a CUDA graph (torch.cuda.CUDAGraph) and replayed.

Every launch of the call is stream-ordered and takes its tensor maps and parameters
by value, so a captured call replays on whatever the input buffers hold at replay
time.  Short sequences are launch-bound, and graphs remove that cost.
"""
import numpy as np
import pytest
import torch

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


def _draw(w, seed):
    return [x.cuda() for x in wl.generate(wl.custom(w.name, w.B, w.H, w.N_q, w.N_kv, w.d, w.causal,
                                                    recipe=w.recipe, H_kv=w.H_kv, seed=seed))]


@pytest.mark.parametrize("pv", ["fp8", "fp16"])
def test_captured_forward_replays_on_new_inputs(pv):
    w = wl.custom("graph", 1, 8, 1000, 1000, 128, True, recipe="llm", H_kv=2, seed=9700)
    q, k, v = _draw(w, 9700)
    ws = sage.make_workspace(1, 8, 1000, 1000, 128, H_kv=2, pv_fp16=(pv == "fp16"))
    out = torch.empty_like(q)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):   # warm-up outside the capture (attributes, module load)
        sage.attn_fwd(q, k, v, causal=True, out=out, workspace=ws, pv=pv)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        sage.attn_fwd(q, k, v, causal=True, out=out, workspace=ws, pv=pv)
    for seed in (9701, 9702):
        qn, kn, vn = _draw(w, seed)
        q.copy_(qn)
        k.copy_(kn)
        v.copy_(vn)
        g.replay()
        torch.cuda.synchronize()
        ref = sage.attn_fwd(qn, kn, vn, causal=True, pv=pv)
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
    assert sage.get_device_status(ws) == (0, 0)


def test_captured_varlen_forward():
    lq = [300, 1, 700, 129]
    H, Hk, d = 4, 2, 64
    g0 = torch.Generator().manual_seed(9800)
    tq = sum(lq)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lq)]), dtype=torch.int32).cuda()

    def draw():
        q = torch.randn(tq, H, d, generator=g0).to(torch.bfloat16).cuda()
        k = (torch.randn(tq, Hk, d, generator=g0) + 2).to(torch.bfloat16).cuda()
        v = torch.randn(tq, Hk, d, generator=g0).to(torch.bfloat16).cuda()
        return q, k, v

    q, k, v = draw()
    ws = sage.make_workspace(len(lq), H, max(lq), max(lq), d, H_kv=Hk)
    out = torch.empty_like(q)
    kw = dict(max_seqlen_q=max(lq), max_seqlen_kv=max(lq), causal=True, out=out, workspace=ws)
    sage.attn_fwd_varlen(q, k, v, cu, cu, **kw)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        sage.attn_fwd_varlen(q, k, v, cu, cu, **kw)
    qn, kn, vn = draw()
    q.copy_(qn)
    k.copy_(kn)
    v.copy_(vn)
    g.replay()
    torch.cuda.synchronize()
    ref = sage.attn_fwd_varlen(qn, kn, vn, cu, cu, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
