"""sage_attn_fwd_noalloc: the forward for callers that cannot allocate device memory
(and so cannot hand the library a workspace), with its scratch in a fixed device
array inside the library.  Checked through the C ABI against sage_attn_fwd, the
entry point that takes a caller-owned workspace, on two calls in a row: both run the
same kernels on the same workspace layout, so the outputs are bit-identical.

This file is collected last on purpose, and passes both alone in a fresh process
and after the rest of the suite."""
import ctypes

import numpy as np
import pytest
import torch

import quantized_attention_fine_b200 as sage
from quantized_attention_fine_b200 import workloads as wl

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 64 << 20


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from quantized_attention_fine_b200 import _build
    _build.build()
    lib = sage.load_library()
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.sage_attn_fwd_noalloc.argtypes = [P, P, P, P, I, I, I, I, I, I, I, I, F, ctypes.POINTER(sage.QuantMode), P]
    lib.sage_attn_fwd_noalloc.restype = I
    lib.sage_noalloc_get_device_status.argtypes = [P, ctypes.POINTER(I), ctypes.POINTER(I)]
    lib.sage_noalloc_get_device_status.restype = I
    return lib


def _status(lib):
    code, site = ctypes.c_int(-1), ctypes.c_int(-1)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.sage_noalloc_get_device_status(stream, ctypes.byref(code), ctypes.byref(site)) == 0
    return code.value, site.value


def _call_noalloc(lib, q, k, v, o, causal, mode):
    B, H, nq, d = q.shape
    nk = k.shape[2]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.sage_attn_fwd_noalloc(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                                     ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(o.data_ptr()),
                                     1 if q.dtype == torch.bfloat16 else 0, 0, B, H, nq, nk, d, int(causal), 0.0,
                                     ctypes.byref(mode), stream)


def test_noalloc_matches_workspace_entry_point_on_two_calls(lib):
    mode = sage.QuantMode.make()
    cases = [wl.custom("noalloc_a", 1, 4, 700, 700, 128, True, recipe="llm", seed=4242),
             wl.custom("noalloc_b", 2, 3, 513, 900, 64, False, recipe="video_dit", seed=4343)]
    for w in cases:
        q, k, v = (x.cuda() for x in wl.generate(w))
        assert sage.workspace_bytes(w.B, w.H, w.N_q, w.N_kv, w.d) <= SCRATCH_BYTES - 1024
        ref = sage.attn_fwd(q, k, v, causal=w.causal)
        o = torch.full_like(q, float("nan"))
        assert _call_noalloc(lib, q, k, v, o, w.causal, mode) == 0
        torch.cuda.synchronize()
        assert torch.equal(o, ref), w.name
        assert _status(lib) == (0, 0)


def test_noalloc_refuses_problems_larger_than_its_scratch(lib):
    # B=1, H=32, N=8192, d=128 needs more than 64 MiB of workspace
    B, H, n, d = 1, 32, 8192, 128
    assert sage.workspace_bytes(B, H, n, n, d) > SCRATCH_BYTES
    q = torch.zeros((B, H, 128, d), dtype=torch.bfloat16, device="cuda")
    o = torch.full_like(q, 3.0)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    ptr = ctypes.c_void_p(q.data_ptr())
    rc = lib.sage_attn_fwd_noalloc(ptr, ptr, ptr, ctypes.c_void_p(o.data_ptr()), 1, 0, B, H, n, n, d, 0, 0.0,
                                   None, stream)
    torch.cuda.synchronize()
    assert rc == sage.SAGE_ERR_WORKSPACE
    assert torch.all(o == 3.0)      # nothing was enqueued


def test_noalloc_fp16_pv_mode(lib):
    """The FP16 P / V mode sizes its scratch with its own (larger) workspace and matches
    the workspace entry point."""
    w = wl.custom("noalloc_pv16", 1, 4, 600, 600, 128, True, recipe="llm", seed=4444)
    q, k, v = (x.cuda() for x in wl.generate(w))
    mode = sage.QuantMode.make(pv="fp16")
    assert sage.workspace_bytes(1, 4, 600, 600, 128, pv_fp16=True) > sage.workspace_bytes(1, 4, 600, 600, 128)
    ref = sage.attn_fwd(q, k, v, causal=True, pv="fp16")
    o = torch.full_like(q, float("nan"))
    assert _call_noalloc(lib, q, k, v, o, True, mode) == 0
    torch.cuda.synchronize()
    assert torch.equal(o, ref)


def test_noalloc_reports_a_device_timeout_and_recovers(lib):
    """A bounded wait that runs out inside the scratch array's kernels is reported by
    sage_noalloc_get_device_status (read and clear), and the next call is correct.  The
    timeout is made on the host side: the attention kernel runs on the array with one
    producer signal withheld (no trap, no fault, no hang)."""
    w = wl.custom("noalloc_to", 1, 2, 256, 256, 64, False, recipe="tiny", seed=4545)
    q, k, v = (x.cuda() for x in wl.generate(w))
    mode = sage.QuantMode.make()
    o = torch.empty_like(q)
    assert _call_noalloc(lib, q, k, v, o, False, mode) == 0
    assert _status(lib) == (0, 0)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    o2 = torch.zeros_like(q)
    rc = lib.sage_debug_attn_fault_inject(ctypes.c_void_p(o2.data_ptr()), 0 if q.dtype == torch.float16 else 1, 0,
                                          w.B, w.H, w.N_q, w.N_kv, w.d, 0, None, 0, stream)
    assert rc == 0
    code, site = _status(lib)
    assert code == sage.SAGE_ERR_TIMEOUT and site != 0
    assert _status(lib) == (0, 0)
    ref = sage.attn_fwd(q, k, v, causal=False)
    o3 = torch.full_like(q, float("nan"))
    assert _call_noalloc(lib, q, k, v, o3, False, mode) == 0
    torch.cuda.synchronize()
    assert torch.equal(o3, ref)
    assert _status(lib) == (0, 0)


def test_noalloc_argument_errors_enqueue_nothing(lib):
    """A call with a bad dtype, mode or size on a capturing stream returns its error and
    leaves the captured graph empty; a B = 0 call (the initialisation call) does too."""
    from cuda.bindings import runtime as cudart
    q = torch.zeros((1, 2, 128, 64), dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    ptr, optr = ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(o.data_ptr())
    bad_mode = sage.QuantMode.make()
    bad_mode.gran = 9
    s = torch.cuda.Stream()
    torch.cuda.synchronize()
    err, = cudart.cudaStreamBeginCapture(s.cuda_stream, cudart.cudaStreamCaptureMode.cudaStreamCaptureModeRelaxed)
    assert err == cudart.cudaError_t.cudaSuccess
    h = ctypes.c_void_p(s.cuda_stream)
    rcs = [lib.sage_attn_fwd_noalloc(ptr, ptr, ptr, optr, 7, 0, 1, 2, 128, 128, 64, 0, 0.0, None, h),
           lib.sage_attn_fwd_noalloc(ptr, ptr, ptr, optr, 1, 0, 1, 2, 128, 128, 64, 0, 0.0, ctypes.byref(bad_mode), h),
           lib.sage_attn_fwd_noalloc(ptr, ptr, ptr, optr, 1, 0, 1, 2, 128, 128, 96, 0, 0.0, None, h),
           lib.sage_attn_fwd_noalloc(ptr, ptr, ptr, optr, 1, 0, 1, 32, 8192, 8192, 128, 0, 0.0, None, h),
           lib.sage_attn_fwd_noalloc(None, None, None, None, 1, 0, 0, 2, 128, 128, 64, 0, 0.0, None, h)]
    err, graph = cudart.cudaStreamEndCapture(s.cuda_stream)
    assert err == cudart.cudaError_t.cudaSuccess
    err, _, n_nodes = cudart.cudaGraphGetNodes(graph, 0)
    assert err == cudart.cudaError_t.cudaSuccess
    cudart.cudaGraphDestroy(graph)
    assert rcs == [sage.SAGE_ERR_INVALID_ARG, sage.SAGE_ERR_INVALID_ARG, sage.SAGE_ERR_UNSUPPORTED,
                   sage.SAGE_ERR_WORKSPACE, 0]
    assert n_nodes == 0
