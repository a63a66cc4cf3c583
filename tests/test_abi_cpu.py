"""Host-side checks of the C ABI that need no GPU: the library loads, exports every
symbol include/sage.h declares, sizes its workspace consistently, and rejects bad
arguments synchronously (before any CUDA call)."""
import ctypes
import os
import re

import pytest

import quantized_attention_fine_b200 as sage
from quantized_attention_fine_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sage.h")


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return sage.load_library()


def _declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"SAGE_API\s+[\w\s\*]+?\b(sage_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = _declared_symbols()
    for required in ("sage_workspace_bytes", "sage_quant_qk", "sage_quant_v", "sage_attn_fwd",
                     "sage_attn_fwd_prequant", "sage_get_device_status"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in _declared_symbols() if not hasattr(lib, n)]
    assert not missing, missing


def test_library_hides_internal_symbols(lib):
    # only the C ABI is exported (built with -fvisibility=hidden)
    for internal in ("_ZN4sage14launch_prepassERKNS_11PrepassArgsEiiP11CUstream_st", "launch_prepass"):
        with pytest.raises(AttributeError):
            getattr(lib, internal)


def test_version_string(lib):
    assert b"sm_100a" in lib.sage_version()


@pytest.mark.parametrize("dims", [(1, 2, 256, 256, 64), (2, 16, 4096, 4096, 128), (1, 32, 32768, 32768, 128),
                                  (2, 48, 17776, 17776, 64), (1, 1, 1, 1, 64), (3, 5, 200, 333, 128)])
def test_workspace_layout_regions_are_aligned_and_disjoint(lib, dims):
    B, H, nq, nk, d = dims
    total = sage.workspace_bytes(*dims)
    BH, Tq = B * H, -(-nq // 128)
    nq_pad, nk_pad = Tq * 128, -(-nk // 128) * 128
    sizes = {0: BH * nq_pad * d, 1: BH * nk_pad * d, 2: BH * d * nk_pad, 3: BH * nq_pad * 4,
             4: BH * nk_pad // 16 * 4, 5: BH * d * 4, 6: BH * Tq * d * 4, 7: BH * d * 4, 8: BH * Tq * nk_pad * 4,
             9: BH * nq_pad * 4, 10: BH * nq_pad * 4}
    spans = []
    for which, size in sizes.items():
        off = lib.sage_workspace_offset(B, H, nq, nk, d, which)
        assert off >= 256 and off % 1024 == 0
        spans.append((off, off + size))
    spans.sort()
    for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
        assert a1 <= b0
    assert spans[-1][1] <= total


@pytest.mark.parametrize("dims", [(1, 8, 2, 256, 300, 64), (2, 32, 8, 4096, 4096, 128), (1, 6, 1, 1, 129, 128)])
def test_gqa_workspace_regions_sized_per_kv_head(lib, dims):
    """Per-query-head regions take B*H rows, per-key/value-head regions B*H_kv."""
    B, H, Hk, nq, nk, d = dims
    total = sage.workspace_bytes(B, H, nq, nk, d, H_kv=Hk)
    assert 0 < total < sage.workspace_bytes(B, H, nq, nk, d)
    BH, BHk, Tq = B * H, B * Hk, -(-nq // 128)
    nq_pad, nk_pad = Tq * 128, -(-nk // 128) * 128
    sizes = {0: BH * nq_pad * d, 1: BHk * nk_pad * d, 2: BHk * d * nk_pad, 3: BH * nq_pad * 4,
             4: BHk * nk_pad // 16 * 4, 5: BHk * d * 4, 6: BH * Tq * d * 4, 7: BHk * d * 4, 8: BH * Tq * nk_pad * 4,
             9: BH * nq_pad * 4, 10: BH * nq_pad * 4}
    spans = []
    for which, size in sizes.items():
        off = lib.sage_workspace_offset_gqa(B, H, Hk, nq, nk, d, which)
        assert off >= 256 and off % 1024 == 0
        spans.append((off, off + size))
    spans.sort()
    for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
        assert a1 <= b0
    assert spans[-1][1] <= total
    # the multi-head entry points are the H_kv = H case
    assert lib.sage_workspace_bytes_gqa(B, H, H, nq, nk, d) == lib.sage_workspace_bytes(B, H, nq, nk, d)


def test_gqa_head_counts_validated(lib):
    assert lib.sage_workspace_bytes_gqa(1, 6, 4, 128, 128, 64) == 0    # 4 does not divide 6
    assert lib.sage_workspace_bytes_gqa(1, 6, 0, 128, 128, 64) == 0
    assert lib.sage_workspace_bytes_gqa(1, 2, 4, 128, 128, 64) == 0    # more key/value heads than query heads
    assert lib.sage_workspace_bytes_gqa(1, 6, 3, 128, 128, 64) > 0
    fake = ctypes.c_void_p(1 << 20)
    assert lib.sage_attn_fwd_gqa(fake, fake, fake, fake, 1, 0, 1, 6, 4, 128, 128, 64, 0, 0.0, None, fake, 1 << 30,
                                 None) == 1


def test_fp16_pv_mode_workspace(lib):
    """The FP16 P / V mode keeps 2 bytes per transposed V element; the other regions move
    up accordingly.  A bad pv_fp16 value is refused."""
    B, H, Hk, nq, nk, d = 1, 4, 2, 300, 520, 128
    m8, m16 = sage.QuantMode.make(), sage.QuantMode.make(pv="fp16")
    b8 = lib.sage_workspace_bytes_mode(B, H, Hk, nq, nk, d, ctypes.byref(m8))
    b16 = lib.sage_workspace_bytes_mode(B, H, Hk, nq, nk, d, ctypes.byref(m16))
    assert b8 == lib.sage_workspace_bytes_gqa(B, H, Hk, nq, nk, d)
    nk_pad = -(-nk // 128) * 128
    assert b16 >= b8 + B * Hk * d * nk_pad - 1024
    o8 = lib.sage_workspace_offset_mode(B, H, Hk, nq, nk, d, ctypes.byref(m8), 2)
    o16 = lib.sage_workspace_offset_mode(B, H, Hk, nq, nk, d, ctypes.byref(m16), 2)
    assert o8 == o16   # V^T itself starts at the same place
    ds8 = lib.sage_workspace_offset_mode(B, H, Hk, nq, nk, d, ctypes.byref(m8), 8)
    ds16 = lib.sage_workspace_offset_mode(B, H, Hk, nq, nk, d, ctypes.byref(m16), 8)
    assert ds16 - ds8 >= B * Hk * d * nk_pad - 1024
    bad = sage.QuantMode.make()
    bad.pv_fp16 = 2
    assert lib.sage_workspace_bytes_mode(B, H, Hk, nq, nk, d, ctypes.byref(bad)) == 0


def test_workspace_bytes_rejects_bad_sizes(lib):
    assert lib.sage_workspace_bytes(1, 1, 128, 128, 96) == 0      # d must be 64 or 128
    assert lib.sage_workspace_bytes(-1, 1, 128, 128, 64) == 0
    assert lib.sage_workspace_bytes(1 << 16, 1 << 10, 1 << 12, 128, 64) == 0   # beyond 32-bit TMA coordinates
    assert lib.sage_workspace_offset(1, 1, 128, 128, 64, 99) == -1


def test_argument_errors_return_synchronously(lib):
    P = ctypes.c_void_p
    fake = P(1 << 20)  # never dereferenced: validation fails first
    # bad dtype / layout / d / null pointers
    assert lib.sage_attn_fwd(fake, fake, fake, fake, 7, 0, 1, 1, 128, 128, 64, 0, 0.0, None, fake, 1 << 30, None) == 1
    assert lib.sage_attn_fwd(fake, fake, fake, fake, 1, 3, 1, 1, 128, 128, 64, 0, 0.0, None, fake, 1 << 30, None) == 1
    assert lib.sage_attn_fwd(fake, fake, fake, fake, 1, 0, 1, 1, 128, 128, 80, 0, 0.0, None, fake, 1 << 30, None) == 2
    assert lib.sage_attn_fwd(None, fake, fake, fake, 1, 0, 1, 1, 128, 128, 64, 0, 0.0, None, fake, 1 << 30, None) == 1
    # misaligned input
    assert lib.sage_attn_fwd(P((1 << 20) + 2), fake, fake, fake, 1, 0, 1, 1, 128, 128, 64, 0, 0.0, None, fake,
                             1 << 30, None) == 2
    # workspace too small / misaligned
    assert lib.sage_attn_fwd(fake, fake, fake, fake, 1, 0, 1, 1, 128, 128, 64, 0, 0.0, None, fake, 16, None) == 3
    assert lib.sage_attn_fwd(fake, fake, fake, fake, 1, 0, 1, 1, 128, 128, 64, 0, 0.0, None, P((1 << 20) + 512),
                             1 << 30, None) == 2
    # bad quant modes
    bad = sage.QuantMode(9, 1, 1, 448.0, 448.0)
    assert lib.sage_quant_qk(fake, fake, 1, 0, 1, 1, 128, 128, 64, ctypes.byref(bad), fake, 1 << 30, None) == 1
    bad = sage.QuantMode(2, 1, 1, 500.0, 448.0)
    assert lib.sage_quant_v(fake, 1, 0, 1, 1, 128, 128, 64, ctypes.byref(bad), fake, 1 << 30, None) == 1
    # empty problems are a successful no-op
    assert lib.sage_attn_fwd(fake, fake, fake, fake, 1, 0, 0, 4, 128, 128, 64, 0, 0.0, None, None, 0, None) == 0
    assert lib.sage_attn_fwd(fake, fake, fake, fake, 1, 0, 1, 4, 0, 128, 64, 0, 0.0, None, None, 0, None) == 0
    # diagnostics validate their indices
    assert lib.sage_debug_qk_tile(fake, 1, 1, 128, 128, 64, 1, 0, 0, fake, None) == 1
    assert lib.sage_debug_pv_accumulate(fake, fake, 0, 64, fake, None) == 1
    assert lib.sage_debug_quotient_check(fake, 0, 1, fake, fake, None) == 1
    assert lib.sage_debug_quotient_check(fake, 4, 7, fake, fake, None) == 1
    assert lib.sage_debug_quotient_check(None, 4, 1, fake, fake, None) == 1


def test_noalloc_argument_errors_come_before_any_cuda_call(lib):
    """sage_attn_fwd_noalloc checks its arguments as sage_attn_fwd does before it
    touches CUDA: with no GPU here, any CUDA call would turn the result into
    SAGE_ERR_CUDA, so the exact statuses show that nothing was enqueued."""
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    fn = lib.sage_attn_fwd_noalloc
    fn.argtypes = [P, P, P, P, I, I, I, I, I, I, I, I, F, ctypes.POINTER(sage.QuantMode), P]
    fn.restype = I
    fake = P(1 << 20)
    assert fn(fake, fake, fake, fake, 7, 0, 1, 1, 128, 128, 64, 0, 0.0, None, None) == 1      # dtype
    assert fn(fake, fake, fake, fake, 1, 3, 1, 1, 128, 128, 64, 0, 0.0, None, None) == 1      # layout
    assert fn(fake, fake, fake, fake, 1, 0, 1, 1, 128, 128, 80, 0, 0.0, None, None) == 2      # d
    assert fn(None, fake, fake, fake, 1, 0, 1, 1, 128, 128, 64, 0, 0.0, None, None) == 1      # null q
    assert fn(P((1 << 20) + 2), fake, fake, fake, 1, 0, 1, 1, 128, 128, 64, 0, 0.0, None, None) == 2
    bad = sage.QuantMode(9, 1, 1, 448.0, 448.0)
    assert fn(fake, fake, fake, fake, 1, 0, 1, 1, 128, 128, 64, 0, 0.0, ctypes.byref(bad), None) == 1
    # beyond 32-bit TMA coordinates: the unsupported-size status of sage_attn_fwd
    assert fn(fake, fake, fake, fake, 1, 0, 1 << 16, 1 << 10, 1 << 12, 128, 64, 0, 0.0, None, None) == 2
    assert lib.sage_noalloc_get_device_status(None, None, None) == 1


def test_python_binding_has_no_fallback(monkeypatch, tmp_path):
    monkeypatch.setattr(sage, "_LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(sage, "_lib", None)
    with pytest.raises(RuntimeError, match="not built"):
        sage.load_library()


def test_varlen_and_mode_argument_errors_return_synchronously(lib):
    """Argument checks of the packed-batch entry point and of the quantization mode:
    each returns before any CUDA call (so they run here, without a GPU)."""
    P, I = ctypes.c_void_p, ctypes.c_int
    fake = P(1 << 20)
    assert lib.sage_workspace_bytes_varlen(3, 8, 2, 700, 900, 128) == lib.sage_workspace_bytes_gqa(3, 8, 2, 700, 900,
                                                                                                   128)
    f = lib.sage_attn_fwd_varlen
    args = lambda **kw: [kw.get("q", fake), fake, fake, fake, kw.get("dtype", 1), kw.get("cu_q", fake),
                         kw.get("cu_kv", fake), kw.get("B", 2), 8, kw.get("Hk", 2), kw.get("tq", 100),
                         kw.get("tk", 100), 64, 64, kw.get("d", 64), 1, 0.0, kw.get("mode", None), fake, 1 << 30,
                         None]
    assert f(*args(cu_q=None)) == 1                     # offsets are required
    assert f(*args(cu_kv=None)) == 1
    assert f(*args(tq=-1)) == 1                         # negative totals
    assert f(*args(Hk=3)) == 1                          # 3 does not divide 8
    assert f(*args(d=96)) == 2                          # head dim
    assert f(*args(dtype=5)) == 1                       # dtype
    assert f(*args(q=P((1 << 20) + 4))) == 2            # misaligned
    assert f(*args(B=0)) == 0 and f(*args(tq=0)) == 0   # nothing to do
    bad = sage.QuantMode.make()
    bad.pv_fp16 = 3
    assert f(*args(mode=ctypes.byref(bad))) == 1
    bad = sage.QuantMode.make()
    bad.p_range = 500.0                                 # beyond the E4M3 range
    assert f(*args(mode=ctypes.byref(bad))) == 1


def test_in_kernel_q_entry_points_check_arguments_before_any_cuda_call(lib):
    """The entry points that quantize Q inside the attention kernel check their arguments
    as sage_attn_fwd does, before any CUDA call (with no GPU here a CUDA call would turn
    the result into SAGE_ERR_CUDA), and refuse the 4-bit mode, whose Q is quantized in
    the pre-pass."""
    P, I, F, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    fn = lib.sage_attn_fwd_qfused_gqa
    fn.argtypes = [P, P, P, P, I, I, I, I, I, I, I, I, I, F, ctypes.POINTER(sage.QuantMode), P, S, P]
    fn.restype = I
    fake = P(1 << 20)
    assert fn(fake, fake, fake, fake, 7, 0, 1, 2, 2, 128, 128, 64, 0, 0.0, None, fake, 1 << 30, None) == 1   # dtype
    assert fn(fake, fake, fake, fake, 1, 0, 1, 3, 2, 128, 128, 64, 0, 0.0, None, fake, 1 << 30, None) == 1   # heads
    assert fn(None, fake, fake, fake, 1, 0, 1, 2, 2, 128, 128, 64, 0, 0.0, None, fake, 1 << 30, None) == 1   # null q
    assert fn(fake, fake, fake, fake, 1, 0, 1, 2, 2, 128, 128, 80, 0, 0.0, None, fake, 1 << 30, None) == 2   # d
    fp4 = sage.QuantMode.make("fp4")
    assert fn(fake, fake, fake, fake, 1, 0, 1, 2, 2, 128, 128, 64, 0, 0.0, ctypes.byref(fp4), fake, 1 << 30,
              None) == 2
    # v = NULL (the attention only) passes the same checks; a workspace too small is refused
    assert fn(fake, fake, None, fake, 1, 0, 1, 2, 2, 128, 128, 64, 0, 0.0, None, fake, 16, None) == 3
    vfn = lib.sage_attn_fwd_varlen_qfused
    vfn.argtypes = [P, P, P, P, I, P, P] + [I] * 9 + [F, ctypes.POINTER(sage.QuantMode), P, S, P]
    vfn.restype = I
    assert vfn(fake, fake, fake, fake, 1, fake, fake, 1, 2, 2, 128, 128, 128, 128, 64, 0, 0.0, ctypes.byref(fp4),
               fake, 1 << 30, None) == 2
    dump = lib.sage_debug_set_q_code_dump
    dump.argtypes = [I]
    dump.restype = I
    assert dump(2) == 1 and dump(-1) == 1
    assert dump(0) == 0
