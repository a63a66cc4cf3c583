"""Smoothed-INT8-QK / FP8-PV quantized attention forward for NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI of ``libsage_b200.so`` (declared in
``include/sage.h``).  Every step of the computation runs in the library's CUDA
kernels; this module only marshals arguments: torch tensors supply device memory
and the current CUDA stream.  There is no CPU fallback: if the library is missing
every call raises.

    import torch, quantized_attention_fine_b200 as sage
    o = sage.attn_fwd(q, k, v, causal=True)          # q, k, v: [B, H, N, d] bf16/fp16
    o = sage.attn_fwd(q, k, v, layout="NHD")         # [B, N, H, d]
    o = sage.attn_fwd(q, k_gqa, v_gqa)               # k, v with H_kv heads, H_kv | H
    o, lse = sage.attn_fwd(q, k, v, return_lse=True) # row log-sum-exp [B, H, N_q]
    o = sage.attn_fwd(q, k, v, pv="fp16")            # the qk_int8_pv_fp16 mode
    o = sage.attn_fwd_varlen(q_packed, k_packed, v_packed, cu_q, cu_kv, causal=True)
    attn = sage.SageAttention(head_dim=128, is_causal=True, quant_mode="qk_int8_pv_fp8")
    o = attn(q, k, v)                                # drop-in for a model's attention call

Workspaces (sage.make_workspace) can be kept across calls; a whole call can be
captured in a CUDA graph.

Method: "SageAttention2" (arXiv 2411.10958) with the per-channel FP8 V scaling and
P range of SageAttention2++ (arXiv 2505.21136); see include/sage.h.
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

__all__ = [
    "QuantMode", "Workspace", "workspace_bytes", "make_workspace", "quant_qk", "quant_v", "attn_fwd_prequant",
    "attn_fwd", "attn_fwd_varlen", "SageAttention", "scaled_dot_product_attention", "QUANT_MODES", "get_device_status", "workspace_view", "debug_qk_tile", "debug_pv_accumulate",
    "debug_fault_inject", "debug_pv_accumulate_f16acc", "debug_mma_rate", "debug_quant_fp4", "debug_quotient_check", "library_path", "load_library", "SageError", "GRANULARITIES",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libsage_b200.so")
_lock = threading.Lock()
_lib = None

SAGE_OK, SAGE_ERR_INVALID_ARG, SAGE_ERR_UNSUPPORTED, SAGE_ERR_WORKSPACE, SAGE_ERR_CUDA, SAGE_ERR_TIMEOUT = range(6)
_ERR_NAMES = {0: "SAGE_OK", 1: "SAGE_ERR_INVALID_ARG", 2: "SAGE_ERR_UNSUPPORTED", 3: "SAGE_ERR_WORKSPACE",
              4: "SAGE_ERR_CUDA", 5: "SAGE_ERR_TIMEOUT"}
GRANULARITIES = {"per_block": 0, "per_warp": 1, "per_threadgroup": 2, "fp4": 3}
QK_FP4 = 3   # granularity code of the 4-bit Q / K mode (SAGE_QK_FP4)
_LAYOUTS = {"HND": 0, "NHD": 1}
WS_VIEWS = {"q8": 0, "k8": 1, "vt8": 2, "dq": 3, "dk": 4, "dv": 5, "qbar": 6, "kbar": 7, "ds": 8, "qs_kbar": 9,
            "lse": 10, "sfq": 11, "sfk": 12}
WS_ALIGN = 1024


class SageError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__("%s failed: %s (%d)" % (what, _ERR_NAMES.get(code, "?"), code))
        self.code = code


class QuantMode(ctypes.Structure):
    """Mirror of sage_quant_mode_t."""
    _fields_ = [("gran", ctypes.c_int32), ("smooth_q", ctypes.c_int32), ("smooth_k", ctypes.c_int32),
                ("p_range", ctypes.c_float), ("v_range", ctypes.c_float), ("pv_fp16", ctypes.c_int32)]

    @classmethod
    def make(cls, granularity="per_threadgroup", smooth_q=True, smooth_k=True, p_range=448.0, v_range=448.0,
             pv="fp8"):
        """pv: "fp8" (E4M3 P and per-channel E4M3 V, the default) or "fp16" (FP16 P~ and V,
        the "qk_int8_pv_fp16" high-fidelity mode)."""
        g = GRANULARITIES[granularity] if isinstance(granularity, str) else int(granularity)
        if pv not in ("fp8", "fp16"):
            raise ValueError("pv must be 'fp8' or 'fp16'")
        return cls(g, int(bool(smooth_q)), int(bool(smooth_k)), float(p_range), float(v_range), int(pv == "fp16"))


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load libsage_b200.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError("libsage_b200.so is not built (run `python -m quantized_attention_fine_b200._build`); "
                               "there is no fallback implementation")
        lib = ctypes.CDLL(_LIB_PATH)
        P, I, F, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        QM = ctypes.POINTER(QuantMode)
        lib.sage_workspace_bytes.argtypes = [I] * 5
        lib.sage_workspace_bytes.restype = S
        lib.sage_workspace_offset.argtypes = [I] * 6
        lib.sage_workspace_offset.restype = ctypes.c_int64
        lib.sage_quant_qk.argtypes = [P, P, I, I, I, I, I, I, I, QM, P, S, P]
        lib.sage_quant_v.argtypes = [P, I, I, I, I, I, I, I, QM, P, S, P]
        lib.sage_attn_fwd_prequant.argtypes = [P, I, I, I, I, I, I, I, I, F, QM, P, S, P]
        lib.sage_attn_fwd.argtypes = [P, P, P, P, I, I, I, I, I, I, I, I, F, QM, P, S, P]
        lib.sage_workspace_bytes_gqa.argtypes = [I] * 6
        lib.sage_workspace_bytes_gqa.restype = S
        lib.sage_workspace_bytes_mode.argtypes = [I] * 6 + [QM]
        lib.sage_workspace_bytes_mode.restype = S
        lib.sage_workspace_offset_mode.argtypes = [I] * 6 + [QM, I]
        lib.sage_workspace_offset_mode.restype = ctypes.c_int64
        lib.sage_workspace_offset_gqa.argtypes = [I] * 7
        lib.sage_workspace_offset_gqa.restype = ctypes.c_int64
        lib.sage_quant_qk_gqa.argtypes = [P, P, I, I, I, I, I, I, I, I, QM, P, S, P]
        lib.sage_quant_v_gqa.argtypes = [P, I, I, I, I, I, I, I, I, QM, P, S, P]
        lib.sage_attn_fwd_prequant_gqa.argtypes = [P, I, I, I, I, I, I, I, I, I, F, QM, P, S, P]
        lib.sage_attn_fwd_gqa.argtypes = [P, P, P, P, I, I, I, I, I, I, I, I, I, F, QM, P, S, P]
        lib.sage_workspace_bytes_varlen.argtypes = [I] * 6
        lib.sage_workspace_bytes_varlen.restype = S
        lib.sage_attn_fwd_varlen.argtypes = [P, P, P, P, I, P, P] + [I] * 9 + [F, QM, P, S, P]
        lib.sage_get_device_status.argtypes = [P, P, ctypes.POINTER(I), ctypes.POINTER(I)]
        lib.sage_debug_qk_tile.argtypes = [P, I, I, I, I, I, I, I, I, P, P]
        lib.sage_debug_pv_accumulate.argtypes = [P, P, I, I, P, P]
        lib.sage_debug_pv_accumulate_f16acc.argtypes = [P, P, I, I, P, P]
        lib.sage_debug_mma_rate.argtypes = [I, I, I, P, P]
        lib.sage_debug_quant_fp4.argtypes = [P, I, I, P, P, P, P]
        lib.sage_debug_quotient_check.argtypes = [P, I, I, P, P, P]
        lib.sage_debug_qk_tile_fp4.argtypes = [P, P, P, P, I, P, P, P]
        lib.sage_debug_attn_fault_inject.argtypes = [P, I, I, I, I, I, I, I, I, P, S, P]
        lib.sage_attn_fwd_qfused_gqa.argtypes = [P, P, P, P, I, I, I, I, I, I, I, I, I, F, QM, P, S, P]
        lib.sage_attn_fwd_varlen_qfused.argtypes = [P, P, P, P, I, P, P] + [I] * 9 + [F, QM, P, S, P]
        lib.sage_debug_set_q_code_dump.argtypes = [I]
        lib.sage_debug_attn_fault_inject_qfused.argtypes = [P, P, P, I, I, I, I, I, I, I, I, P, S, P]
        lib.sage_version.restype = ctypes.c_char_p
        for fn in ("sage_quant_qk", "sage_quant_v", "sage_attn_fwd_prequant", "sage_attn_fwd",
                   "sage_quant_qk_gqa", "sage_quant_v_gqa", "sage_attn_fwd_prequant_gqa", "sage_attn_fwd_gqa",
                   "sage_attn_fwd_varlen",
                   "sage_get_device_status", "sage_debug_qk_tile", "sage_debug_pv_accumulate",
                   "sage_debug_pv_accumulate_f16acc", "sage_debug_mma_rate", "sage_debug_quant_fp4", "sage_debug_quotient_check",
                   "sage_debug_qk_tile_fp4",
                   "sage_debug_attn_fault_inject", "sage_attn_fwd_qfused_gqa", "sage_attn_fwd_varlen_qfused",
                   "sage_debug_set_q_code_dump", "sage_debug_attn_fault_inject_qfused"):
            getattr(lib, fn).restype = ctypes.c_int
        _lib = lib
        return lib


def _check(code: int, what: str):
    if code != SAGE_OK:
        raise SageError(code, what)


def _torch():
    import torch
    return torch


def _stream_handle(stream=None):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return 1
    if t.dtype == torch.float16:
        return 0
    raise TypeError("q, k, v must be bfloat16 or float16, got %s" % t.dtype)


def _shape(q, k, layout):
    """(B, H, H_kv, n_q, n_kv, d) of q and k; k may have fewer heads than q (H_kv divides H)."""
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q, k, v must be 4-D")
    if layout == "HND":
        B, H, n_q, d = q.shape
        H_kv, n_kv = k.shape[1], k.shape[2]
    elif layout == "NHD":
        B, n_q, H, d = q.shape
        n_kv, H_kv = k.shape[1], k.shape[2]
    else:
        raise ValueError("layout must be 'HND' or 'NHD'")
    if k.shape[0] != B or k.shape[3] != d or H_kv < 1 or H % H_kv != 0:
        raise ValueError("k shape %s does not match q %s" % (tuple(k.shape), tuple(q.shape)))
    return int(B), int(H), int(H_kv), int(n_q), int(n_kv), int(d)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _layout_mode(pv_fp16=False, qk_fp4=False):
    """A mode with the workspace layout of these flags (the other fields do not change it)."""
    return QuantMode.make("fp4" if qk_fp4 else "per_threadgroup", pv="fp16" if pv_fp16 else "fp8")


def workspace_bytes(B, H, n_q, n_kv, d, H_kv=None, pv_fp16=False, qk_fp4=False) -> int:
    H_kv = H if H_kv is None else H_kv
    mode = _layout_mode(pv_fp16, qk_fp4)
    return int(load_library().sage_workspace_bytes_mode(B, H, H_kv, n_q, n_kv, d, ctypes.byref(mode)))


class Workspace:
    """Caller-owned device workspace: a zeroed uint8 tensor with a 1024-byte aligned window.

    dims = (B, H, n_q, n_kv, d) with H query heads; H_kv key/value heads (H_kv = H
    for multi-head attention); pv_fp16: laid out for the FP16 P / V mode; qk_fp4: for
    the 4-bit Q / K mode."""

    def __init__(self, B, H, n_q, n_kv, d, device=None, H_kv=None, pv_fp16=False, qk_fp4=False):
        torch = _torch()
        self.dims = (int(B), int(H), int(n_q), int(n_kv), int(d))
        self.H_kv = int(H if H_kv is None else H_kv)
        self.pv_fp16 = bool(pv_fp16)
        self.qk_fp4 = bool(qk_fp4)
        self.nbytes = workspace_bytes(*self.dims, H_kv=self.H_kv, pv_fp16=self.pv_fp16, qk_fp4=self.qk_fp4)
        if self.nbytes == 0:
            raise SageError(SAGE_ERR_UNSUPPORTED, "sage_workspace_bytes")
        self.tensor = torch.zeros(self.nbytes + WS_ALIGN, dtype=torch.uint8, device=device or "cuda")
        base = self.tensor.data_ptr()
        self.offset = (-base) % WS_ALIGN
        self.ptr = base + self.offset

    def fits(self, B, H, n_q, n_kv, d, H_kv=None, pv_fp16=False, qk_fp4=False) -> bool:
        H_kv = H if H_kv is None else H_kv
        return (self.dims == (int(B), int(H), int(n_q), int(n_kv), int(d)) and self.H_kv == int(H_kv)
                and self.pv_fp16 == bool(pv_fp16) and self.qk_fp4 == bool(qk_fp4))

    def lse(self):
        """Row log-sum-exp [B, H, n_q] (fp32, natural log) of the last attention call on
        this workspace; a view into the workspace, overwritten by the next call."""
        B, H, n_q, _, _ = self.dims
        return self.view("lse").view(B, H, -1)[:, :, :n_q]

    def view(self, which: str):
        """Typed view of a workspace region (see include/sage.h, SAGE_WS_*): per query
        head for q8, dq, qbar, ds; per key/value head for k8, vt8, dk, dv, kbar."""
        torch = _torch()
        B, H, n_q, n_kv, d = self.dims
        mode = _layout_mode(self.pv_fp16, self.qk_fp4)
        off = int(load_library().sage_workspace_offset_mode(B, H, self.H_kv, n_q, n_kv, d, ctypes.byref(mode),
                                                            WS_VIEWS[which]))
        BH, BHk, Tq, Tk = B * H, B * self.H_kv, -(-n_q // 128), -(-n_kv // 128)
        nq_pad, nk_pad = Tq * 128, Tk * 128
        qk = ((BH, nq_pad, d // 2), torch.uint8) if self.qk_fp4 else ((BH, nq_pad, d), torch.int8)
        kk = ((BHk, nk_pad, d // 2), torch.uint8) if self.qk_fp4 else ((BHk, nk_pad, d), torch.int8)
        shapes = {"q8": qk, "k8": kk,
                  # E4M3 scale atoms: regions of the 4-bit mode only (empty otherwise)
                  "sfq": ((BH, Tq, d // 64 if self.qk_fp4 else 0, 512), torch.uint8),
                  "sfk": ((BHk, Tk, d // 64 if self.qk_fp4 else 0, 512), torch.uint8),
                  "vt8": ((BHk, d, nk_pad), torch.float16 if self.pv_fp16 else torch.uint8), "dq": ((BH, nq_pad), torch.float32),
                  "dk": ((BHk, nk_pad // 16), torch.float32), "dv": ((BHk, d), torch.float32),
                  "qbar": ((BH, Tq, d), torch.float32), "kbar": ((BHk, d), torch.float32),
                  "ds": ((BH, Tq, nk_pad), torch.float32), "qs_kbar": ((BH, nq_pad), torch.float32),
                  "lse": ((BH, nq_pad), torch.float32)}
        shp, dt = shapes[which]
        n = math.prod(shp) * torch.tensor([], dtype=dt).element_size()
        start = self.offset + off
        return self.tensor[start:start + n].view(dt).view(shp)


def make_workspace(B, H, n_q, n_kv, d, device=None, H_kv=None, pv_fp16=False, qk_fp4=False) -> Workspace:
    return Workspace(B, H, n_q, n_kv, d, device, H_kv=H_kv, pv_fp16=pv_fp16, qk_fp4=qk_fp4)


def _ws_for(ws, B, H, H_kv, n_q, n_kv, d, device, pv_fp16=False, qk_fp4=False):
    if ws is None:
        return Workspace(B, H, n_q, n_kv, d, device, H_kv=H_kv, pv_fp16=pv_fp16, qk_fp4=qk_fp4)
    if not ws.fits(B, H, n_q, n_kv, d, H_kv, pv_fp16, qk_fp4):
        raise ValueError("workspace was made for %s (H_kv %d, pv_fp16 %s, qk_fp4 %s), not %s (H_kv %d, pv_fp16 %s, "
                         "qk_fp4 %s)" % (ws.dims, ws.H_kv, ws.pv_fp16, ws.qk_fp4, (B, H, n_q, n_kv, d), H_kv,
                                         bool(pv_fp16), bool(qk_fp4)))
    return ws


def quant_qk(q, k, *, layout="HND", mode=None, workspace=None, stream=None) -> Workspace:
    B, H, H_kv, n_q, n_kv, d = _shape(q, k, layout)
    mode = mode or QuantMode.make()
    ws = _ws_for(workspace, B, H, H_kv, n_q, n_kv, d, q.device, mode.pv_fp16, mode.gran == QK_FP4)
    _check(load_library().sage_quant_qk_gqa(_ptr(q), _ptr(k), _dtype_code(q), _LAYOUTS[layout], B, H, H_kv, n_q,
                                            n_kv, d, ctypes.byref(mode), ctypes.c_void_p(ws.ptr), ws.nbytes,
                                            _stream_handle(stream)), "sage_quant_qk_gqa")
    return ws


def quant_v(v, *, n_q, H=None, layout="HND", mode=None, workspace=None, stream=None) -> Workspace:
    """V codes and scales into the workspace.  H: query heads (default: those of
    `workspace`, else the heads of v)."""
    if layout == "HND":
        B, H_kv, n_kv, d = v.shape
    else:
        B, n_kv, H_kv, d = v.shape
    if H is None:
        H = workspace.dims[1] if workspace is not None else H_kv
    B, H, H_kv, n_kv, d = int(B), int(H), int(H_kv), int(n_kv), int(d)
    mode = mode or QuantMode.make()
    ws = _ws_for(workspace, B, H, H_kv, n_q, n_kv, d, v.device, mode.pv_fp16, mode.gran == QK_FP4)
    _check(load_library().sage_quant_v_gqa(_ptr(v), _dtype_code(v), _LAYOUTS[layout], B, H, H_kv, n_q, n_kv, d,
                                           ctypes.byref(mode), ctypes.c_void_p(ws.ptr), ws.nbytes,
                                           _stream_handle(stream)), "sage_quant_v_gqa")
    return ws


def attn_fwd_prequant(workspace: Workspace, *, dtype, layout="HND", causal=False, sm_scale=None, mode=None,
                      out=None, stream=None, return_lse=False):
    """Attention from a workspace filled by quant_qk and quant_v.  With return_lse, also
    the rows' log-sum-exp [B, H, n_q] (a view into the workspace, see Workspace.lse)."""
    torch = _torch()
    B, H, n_q, n_kv, d = workspace.dims
    if out is None:
        shape = (B, H, n_q, d) if layout == "HND" else (B, n_q, H, d)
        out = torch.empty(shape, dtype=dtype, device=workspace.tensor.device)
    mode = mode or QuantMode.make()
    if bool(mode.pv_fp16) != workspace.pv_fp16 or (mode.gran == QK_FP4) != workspace.qk_fp4:
        raise ValueError("the mode's pv / qk setting does not match the workspace")
    _check(load_library().sage_attn_fwd_prequant_gqa(_ptr(out), _dtype_code(out), _LAYOUTS[layout], B, H,
                                                     workspace.H_kv, n_q, n_kv, d, int(bool(causal)),
                                                     float(sm_scale or 0.0), ctypes.byref(mode),
                                                     ctypes.c_void_p(workspace.ptr), workspace.nbytes,
                                                     _stream_handle(stream)), "sage_attn_fwd_prequant_gqa")
    return (out, workspace.lse()) if return_lse else out


def attn_fwd_qfused(q, k, workspace: Workspace, *, causal=False, sm_scale=None, layout="HND", mode=None, out=None,
                    stream=None, return_lse=False):
    """The attention half of ``attn_fwd(..., fuse_q=True)``: Q quantized and the dS bias
    formed inside the attention kernel, from q, k and a workspace whose K / V parts hold
    the pre-pass of k and v (quant_qk + quant_v, or an earlier attn_fwd call, with the
    same sizes and mode)."""
    torch = _torch()
    B, H, H_kv, n_q, n_kv, d = _shape(q, k, layout)
    if (B, H, n_q, n_kv, d) != tuple(workspace.dims) or H_kv != workspace.H_kv:
        raise ValueError("q, k do not match the workspace sizes")
    mode = mode or QuantMode.make()
    if bool(mode.pv_fp16) != workspace.pv_fp16 or (mode.gran == QK_FP4) != workspace.qk_fp4:
        raise ValueError("the mode's pv / qk setting does not match the workspace")
    if out is None:
        out = torch.empty_like(q)
    _check(load_library().sage_attn_fwd_qfused_gqa(_ptr(q), _ptr(k), None, _ptr(out), _dtype_code(q), _LAYOUTS[layout],
                                                   B, H, H_kv, n_q, n_kv, d, int(bool(causal)),
                                                   float(sm_scale or 0.0), ctypes.byref(mode),
                                                   ctypes.c_void_p(workspace.ptr), workspace.nbytes,
                                                   _stream_handle(stream)), "sage_attn_fwd_qfused_gqa")
    return (out, workspace.lse()) if return_lse else out


def debug_set_q_code_dump(enable: bool):
    """While enabled, forward calls that quantize Q inside the attention kernel also
    write the Q codes to the workspace's q8 view (process-wide diagnostic switch)."""
    _check(load_library().sage_debug_set_q_code_dump(int(bool(enable))), "sage_debug_set_q_code_dump")


def attn_fwd(q, k, v, *, causal=False, sm_scale=None, layout="HND", granularity="per_threadgroup",
             smooth_q=True, smooth_k=True, p_range=448.0, v_range=448.0, pv="fp8", out=None, workspace=None,
             stream=None, return_lse=False, fuse_q=False):
    """O = quantized attention of q, k, v (pre-pass + fused kernel, enqueued on the current
    stream).  fuse_q: quantize Q inside the attention kernel instead of the pre-pass
    (sage_attn_fwd_qfused_gqa; slower on B200, kept as an alternative).

    k and v may have fewer heads than q (grouped-query attention): query head h
    reads key/value head h // (H // H_kv).  With return_lse, returns (O, LSE), LSE the
    rows' log-sum-exp [B, H, n_q] fp32 (a view into the workspace)."""
    torch = _torch()
    B, H, H_kv, n_q, n_kv, d = _shape(q, k, layout)
    if v.shape != k.shape:
        raise ValueError("v shape %s must equal k shape %s" % (tuple(v.shape), tuple(k.shape)))
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("q, k, v must share a dtype")
    mode = QuantMode.make(granularity, smooth_q, smooth_k, p_range, v_range, pv)
    ws = _ws_for(workspace, B, H, H_kv, n_q, n_kv, d, q.device, mode.pv_fp16, mode.gran == QK_FP4)
    if out is None:
        out = torch.empty_like(q)
    fn = "sage_attn_fwd_qfused_gqa" if fuse_q else "sage_attn_fwd_gqa"
    _check(getattr(load_library(), fn)(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _dtype_code(q),
                                       _LAYOUTS[layout], B, H, H_kv, n_q, n_kv, d, int(bool(causal)),
                                       float(sm_scale or 0.0), ctypes.byref(mode), ctypes.c_void_p(ws.ptr),
                                       ws.nbytes, _stream_handle(stream)), fn)
    return (out, ws.lse()) if return_lse else out


def attn_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_kv, *, max_seqlen_q=None, max_seqlen_kv=None, causal=False,
                    sm_scale=None, granularity="per_threadgroup", smooth_q=True, smooth_k=True, p_range=448.0,
                    v_range=448.0, pv="fp8", out=None, workspace=None, stream=None, return_lse=False, fuse_q=False):
    """Quantized attention of a packed batch of variable-length sequences (fuse_q: Q
    quantized inside the attention kernel, as in ``attn_fwd``).

    q: [total_q, H, d]; k, v: [total_kv, H_kv, d] (H_kv divides H); cu_seqlens_q,
    cu_seqlens_kv: int32 CUDA tensors of B + 1 offsets.  Sequence b is attended on its
    own.  max_seqlen_*: the longest lengths (read from the offsets, which synchronizes,
    when not given).  With return_lse, also the rows' log-sum-exp as a [B, H,
    max_seqlen_q] view into the workspace (row i of sequence b at [b, h, i])."""
    torch = _torch()
    if q.dim() != 3 or k.dim() != 3 or v.shape != k.shape:
        raise ValueError("q must be [total_q, H, d] and k, v [total_kv, H_kv, d]")
    total_q, H, d = (int(x) for x in q.shape)
    total_kv, H_kv = int(k.shape[0]), int(k.shape[1])
    if int(k.shape[2]) != d or H_kv < 1 or H % H_kv != 0:
        raise ValueError("k shape %s does not match q %s" % (tuple(k.shape), tuple(q.shape)))
    for cu in (cu_seqlens_q, cu_seqlens_kv):
        if cu.dtype != torch.int32 or cu.dim() != 1 or not cu.is_cuda:
            raise ValueError("cu_seqlens must be 1-D int32 CUDA tensors")
    B = int(cu_seqlens_q.numel()) - 1
    if B < 0 or int(cu_seqlens_kv.numel()) != B + 1:
        raise ValueError("cu_seqlens_q and cu_seqlens_kv must both hold B + 1 offsets")
    if max_seqlen_q is None:
        max_seqlen_q = int((cu_seqlens_q[1:] - cu_seqlens_q[:-1]).max().item()) if B > 0 else 0
    if max_seqlen_kv is None:
        max_seqlen_kv = int((cu_seqlens_kv[1:] - cu_seqlens_kv[:-1]).max().item()) if B > 0 else 0
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("q, k, v must share a dtype")
    mode = QuantMode.make(granularity, smooth_q, smooth_k, p_range, v_range, pv)
    ws = _ws_for(workspace, B, H, H_kv, max_seqlen_q, max_seqlen_kv, d, q.device, mode.pv_fp16, mode.gran == QK_FP4)
    if out is None:
        out = torch.empty_like(q)
    fn = "sage_attn_fwd_varlen_qfused" if fuse_q else "sage_attn_fwd_varlen"
    _check(getattr(load_library(), fn)(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _dtype_code(q),
                                       _ptr(cu_seqlens_q), _ptr(cu_seqlens_kv), B, H, H_kv, total_q, total_kv,
                                       int(max_seqlen_q), int(max_seqlen_kv), d, int(bool(causal)),
                                       float(sm_scale or 0.0), ctypes.byref(mode), ctypes.c_void_p(ws.ptr),
                                       ws.nbytes, _stream_handle(stream)), fn)
    if return_lse:
        return out, ws.view("lse").view(B, H, -1)[:, :, :max_seqlen_q]
    return out


# The quantization modes the SageAttention deployment guide names (its usage section):
# INT8 Q / K with FP8 or FP16 P and V.
QUANT_MODES = {"qk_int8_pv_fp8": "fp8", "qk_int8_pv_fp16": "fp16"}


class SageAttention:
    """Callable drop-in for a model's attention function, configured once the way the
    SageAttention deployment guide shows (head_dim, is_causal, quant_mode):

        attn = SageAttention(head_dim=128, is_causal=True, quant_mode="qk_int8_pv_fp16")
        o = attn(q, k, v)          # q [B, H, N_q, d], k / v [B, H_kv, N_kv, d]

    tensor_layout "HND" ([B, H, N, d]) or "NHD" ([B, N, H, d]).  The workspace of the
    last shape is kept and reused (one in-flight call per instance)."""

    def __init__(self, head_dim=128, is_causal=False, quant_mode="qk_int8_pv_fp8", tensor_layout="HND",
                 sm_scale=None, granularity="per_threadgroup", smooth_q=True, smooth_k=True):
        if head_dim not in (64, 128):
            raise ValueError("head_dim must be 64 or 128")
        if quant_mode not in QUANT_MODES:
            raise ValueError("quant_mode must be one of %s" % sorted(QUANT_MODES))
        if tensor_layout not in _LAYOUTS:
            raise ValueError("tensor_layout must be 'HND' or 'NHD'")
        if granularity not in GRANULARITIES:
            raise ValueError("granularity must be one of %s" % sorted(GRANULARITIES))
        self.head_dim, self.is_causal, self.quant_mode = head_dim, bool(is_causal), quant_mode
        self.tensor_layout, self.sm_scale, self.granularity = tensor_layout, sm_scale, granularity
        self.smooth_q, self.smooth_k = smooth_q, smooth_k
        self._ws = None

    def __call__(self, q, k, v, return_lse=False):
        if int(q.shape[-1]) != self.head_dim:
            raise ValueError("head dim %d, configured %d" % (int(q.shape[-1]), self.head_dim))
        B, H, H_kv, n_q, n_kv, d = _shape(q, k, self.tensor_layout)
        pv = QUANT_MODES[self.quant_mode]
        fp4 = self.granularity == "fp4"
        if self._ws is None or not self._ws.fits(B, H, n_q, n_kv, d, H_kv, pv == "fp16", fp4) or \
                self._ws.tensor.device != q.device:
            self._ws = Workspace(B, H, n_q, n_kv, d, q.device, H_kv=H_kv, pv_fp16=(pv == "fp16"), qk_fp4=fp4)
        return attn_fwd(q, k, v, causal=self.is_causal, sm_scale=self.sm_scale, layout=self.tensor_layout,
                        granularity=self.granularity, smooth_q=self.smooth_q, smooth_k=self.smooth_k, pv=pv,
                        workspace=self._ws, return_lse=return_lse)


def scaled_dot_product_attention(query, key, value, attn_mask=None, dropout_p=0.0, is_causal=False, scale=None,
                                 enable_gqa=False, quant_mode="qk_int8_pv_fp8"):
    """The quantized forward behind torch.nn.functional.scaled_dot_product_attention's
    signature ([B, H, N, d] tensors, head-major).  Explicit masks and dropout are not
    part of the method and are refused; is_causal is bottom-right aligned when N_q !=
    N_kv (torch aligns top-left there).  K and V may have fewer heads than Q only with
    enable_gqa, as in torch."""
    if attn_mask is not None:
        raise NotImplementedError("explicit attention masks are not supported (use is_causal)")
    if dropout_p != 0.0:
        raise NotImplementedError("dropout is not supported")
    if quant_mode not in QUANT_MODES:
        raise ValueError("quant_mode must be one of %s" % sorted(QUANT_MODES))
    if query.dim() != 4 or key.dim() != 4:
        raise ValueError("query, key, value must be [B, H, N, d]")
    if int(key.shape[1]) != int(query.shape[1]) and not enable_gqa:
        raise ValueError("key has %d heads and query %d: pass enable_gqa=True" % (int(key.shape[1]),
                                                                                  int(query.shape[1])))
    return attn_fwd(query, key, value, causal=is_causal, sm_scale=scale, layout="HND", pv=QUANT_MODES[quant_mode])


def get_device_status(workspace: Workspace, stream=None):
    """(code, site) of the first device-side error since the last call; clears it."""
    code, site = ctypes.c_int(0), ctypes.c_int(0)
    _check(load_library().sage_get_device_status(ctypes.c_void_p(workspace.ptr), _stream_handle(stream),
                                                 ctypes.byref(code), ctypes.byref(site)), "sage_get_device_status")
    return code.value, site.value


def workspace_view(workspace: Workspace, which: str):
    return workspace.view(which)


def debug_qk_tile(workspace: Workspace, bh: int, q_tile: int, kv_tile: int, stream=None):
    """INT32 S tile [128, 128] read back from tensor memory (diagnostic)."""
    torch = _torch()
    B, H, n_q, n_kv, d = workspace.dims
    if workspace.H_kv != H:
        raise ValueError("debug_qk_tile takes a multi-head workspace")
    out = torch.empty((128, 128), dtype=torch.int32, device=workspace.tensor.device)
    _check(load_library().sage_debug_qk_tile(ctypes.c_void_p(workspace.ptr), B, H, n_q, n_kv, d, bh, q_tile,
                                             kv_tile, _ptr(out), _stream_handle(stream)), "sage_debug_qk_tile")
    return out


def debug_pv_accumulate(p_codes, vt_codes, stream=None):
    """sum_t P_t . V_t with FP32 tensor-memory accumulation (diagnostic).
    p_codes: uint8 [T, 128, 128] E4M3; vt_codes: uint8 [T, d, 128] E4M3.  Returns fp32 [128, d]."""
    torch = _torch()
    T, d = int(p_codes.shape[0]), int(vt_codes.shape[1])
    out = torch.empty((128, d), dtype=torch.float32, device=p_codes.device)
    _check(load_library().sage_debug_pv_accumulate(_ptr(p_codes), _ptr(vt_codes), T, d, _ptr(out),
                                                   _stream_handle(stream)), "sage_debug_pv_accumulate")
    return out


def debug_pv_accumulate_f16acc(p_codes, vt_codes, stream=None):
    """sum_t P_t . V_t on the FP8 tensor core with an FP16 accumulator (diagnostic).
    Returns the raw 32-bit tensor-memory words, int32 [128, d]."""
    torch = _torch()
    T, d = int(p_codes.shape[0]), int(vt_codes.shape[1])
    out = torch.empty((128, d), dtype=torch.int32, device=p_codes.device)
    _check(load_library().sage_debug_pv_accumulate_f16acc(_ptr(p_codes), _ptr(vt_codes), T, d, _ptr(out),
                                                          _stream_handle(stream)), "sage_debug_pv_accumulate_f16acc")
    return out


MMA_KINDS = {"e4m3_f32": (0, 32), "e4m3_f16": (1, 32), "s8_s32": (2, 32), "bf16_f32": (3, 16)}


def debug_mma_rate(kind: str, n_iter: int = 8192, n_ctas=None, repeats: int = 5, stream=None):
    """Tensor-core rate of one tcgen05.mma form (M = 128, N = 256; see MMA_KINDS), in
    dense TFLOP/s (TOPS for S8): best of `repeats` timed launches after one warm-up."""
    torch = _torch()
    code, k = MMA_KINDS[kind]
    dev = torch.cuda.current_device()
    if n_ctas is None:
        n_ctas = torch.cuda.get_device_properties(dev).multi_processor_count
    status = torch.zeros(64, dtype=torch.int32, device="cuda")
    s = stream if stream is not None else torch.cuda.current_stream()
    lib = load_library()
    best = float("inf")
    for i in range(repeats + 1):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        _check(lib.sage_debug_mma_rate(code, n_iter, n_ctas, ctypes.c_void_p(status.data_ptr()),
                                       ctypes.c_void_p(s.cuda_stream)), "sage_debug_mma_rate")
        e1.record(s)
        s.synchronize()
        if i > 0:
            best = min(best, e0.elapsed_time(e1))
    if int(status[0].item()) != 0:
        raise SageError(int(status[0].item()), "sage_debug_mma_rate (device wait)")
    flops = n_ctas * n_iter * 2.0 * 128 * 256 * k
    return flops / (best * 1e-3) / 1e12


def debug_quant_fp4(xs, stream=None):
    """FP4 (E2M1) codes with two-level scales of fp32 rows xs [n, d] (diagnostic).
    Returns (codes uint8 [n_pad, d/2], two per byte; sf uint8 [n_pad, d/16] E4M3 codes;
    g fp32 [n_pad/128])."""
    torch = _torch()
    n, d = int(xs.shape[0]), int(xs.shape[1])
    n_pad = -(-n // 128) * 128
    codes = torch.empty((n_pad, d // 2), dtype=torch.uint8, device=xs.device)
    sf = torch.empty((n_pad, d // 16), dtype=torch.uint8, device=xs.device)
    g = torch.empty((n_pad // 128,), dtype=torch.float32, device=xs.device)
    _check(load_library().sage_debug_quant_fp4(_ptr(xs), n, d, _ptr(codes), _ptr(sf), _ptr(g),
                                               _stream_handle(stream)), "sage_debug_quant_fp4")
    return codes, sf, g


def debug_quotient_check(deltas, dtype, stream=None):
    """Mismatches between the quantizers' quotient routine and the IEEE division over
    every finite 16-bit pattern of `dtype` (torch.bfloat16 or torch.float16) and every
    scale in `deltas` (device fp32).  Returns (count, first) with first = (pattern,
    delta index) of one mismatch, or None."""
    torch = _torch()
    count = torch.zeros(1, dtype=torch.int64, device=deltas.device)
    first = torch.zeros(3, dtype=torch.int32, device=deltas.device)
    deltas = deltas.contiguous()
    _check(load_library().sage_debug_quotient_check(_ptr(deltas), int(deltas.numel()), _dtype_code(torch.empty(0, dtype=dtype)),
                                                    _ptr(count), _ptr(first), _stream_handle(stream)),
           "sage_debug_quotient_check")
    c, f = int(count.item()), first.tolist()
    return c, ((f[0] & 0xFFFF, f[1]) if f[2] else None)


def debug_qk_tile_fp4(q4, k4, sfq, sfk, stream=None):
    """One 128 x 128 QK^T tile of the 4-bit mode on the block-scaled tensor core
    (diagnostic).  q4, k4: uint8 [128, d/2] E2M1 codes (channel 2c in the low nibble of
    byte c); sfq, sfk: uint8 [128, d/16] E4M3 scale codes.  Returns fp32 [128, 128]."""
    torch = _torch()
    d = int(q4.shape[1]) * 2
    out = torch.empty((128, 128), dtype=torch.float32, device=q4.device)
    status = torch.zeros(64, dtype=torch.int32, device=q4.device)
    lib = load_library()
    _check(lib.sage_debug_qk_tile_fp4(_ptr(q4), _ptr(k4), _ptr(sfq), _ptr(sfk), d, _ptr(out), _ptr(status),
                                      _stream_handle(stream)), "sage_debug_qk_tile_fp4")
    code, site = ctypes.c_int(), ctypes.c_int()
    _check(lib.sage_get_device_status(_ptr(status), _stream_handle(stream), ctypes.byref(code), ctypes.byref(site)),
           "sage_get_device_status")
    if code.value != SAGE_OK:
        raise SageError(code.value, "sage_debug_qk_tile_fp4 (device site %d)" % site.value)
    return out


def debug_fault_inject_qfused(q, k, workspace: Workspace, out, *, layout="HND", causal=False, stream=None):
    """The same for the attention kernel that quantizes Q itself (q, k: the caller's tensors)."""
    B, H, n_q, n_kv, d = workspace.dims
    if workspace.H_kv != H:
        raise ValueError("debug_fault_inject_qfused takes a multi-head workspace")
    _check(load_library().sage_debug_attn_fault_inject_qfused(_ptr(q), _ptr(k), _ptr(out), _dtype_code(out),
                                                              _LAYOUTS[layout], B, H, n_q, n_kv, d, int(bool(causal)),
                                                              ctypes.c_void_p(workspace.ptr), workspace.nbytes,
                                                              _stream_handle(stream)),
           "sage_debug_attn_fault_inject_qfused")


def debug_fault_inject(workspace: Workspace, out, *, layout="HND", causal=False, stream=None):
    """Run the attention kernel with one producer signal withheld (the bounded wait must run out)."""
    B, H, n_q, n_kv, d = workspace.dims
    if workspace.H_kv != H:
        raise ValueError("debug_fault_inject takes a multi-head workspace")
    _check(load_library().sage_debug_attn_fault_inject(_ptr(out), _dtype_code(out), _LAYOUTS[layout], B, H, n_q,
                                                       n_kv, d, int(bool(causal)), ctypes.c_void_p(workspace.ptr),
                                                       workspace.nbytes, _stream_handle(stream)),
           "sage_debug_attn_fault_inject")
