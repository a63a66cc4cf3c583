"""fp64 CPU oracle of the smoothed-INT8-QK / FP8-PV attention forward.

TEST INFRASTRUCTURE ONLY: the test-suite, the smoke check and the CPU-baseline
leg of ``bench.py`` may import this package; the CUDA product path never does.
It shares no code with the CUDA path.  The arithmetic lives in
``sage_oracle.c`` (plain C, fp64, OpenMP over rows); this module compiles it
with gcc, loads it with ctypes and marshals numpy arrays.

Method sources (page title and section):
  * "SageAttention2: Efficient Attention with Thorough Outlier Smoothing and
    Per-thread INT4 Quantization" (arXiv 2411.10958), abstract -- Q/K smoothing,
    fine-grained Q/K quantization, FP8 (P~, V), two-level PV accumulation.
  * pith.science verdict on arXiv 2505.21136 (SageAttention2++), fields
    key_machinery and core_discovery -- per-channel delta_V = |max V| / Vr,
    P range Pr, the Pr x Vr <= 2047/2 bound of the FP16-accumulator variant.

Parity status of each function is stated in its docstring; the pins live in
``tests/test_oracle_pins.py``.  ``tests/test_oracle_mutations.py`` plants mistakes in
the C code (built with ORACLE_MUTATION = k, selected by the environment variable
SAGE_ORACLE_MUTATION, which nothing else sets) and checks that the pins reject each.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sage_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "libsage_oracle.so")
_lock = threading.Lock()
_lib = None

TILE = 128


def build(force: bool = False, mutation: int = 0) -> str:
    """Compile sage_oracle.c into oracle/_build/libsage_oracle.so (gcc, OpenMP).
    mutation > 0 builds, beside it, the oracle with planted mistake `mutation` (see
    ORACLE_MUTATION in sage_oracle.c); only the pins' own tests use those builds."""
    os.makedirs(_BUILD, exist_ok=True)
    path = _LIB_PATH if mutation == 0 else os.path.join(_BUILD, "libsage_oracle_mut%d.so" % mutation)
    if (not force and os.path.exists(path)
            and os.path.getmtime(path) >= os.path.getmtime(_SRC)):
        return path
    tmp = path + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-ffp-contract=off", "-fno-fast-math", "-DORACLE_MUTATION=%d" % mutation, "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, path)
    return path


class _Cfg(ctypes.Structure):
    _fields_ = [("n_q", ctypes.c_int), ("n_kv", ctypes.c_int), ("d", ctypes.c_int),
                ("g_q", ctypes.c_int), ("g_k", ctypes.c_int),
                ("smooth_q", ctypes.c_int), ("smooth_k", ctypes.c_int),
                ("quant_qk", ctypes.c_int), ("quant_p", ctypes.c_int), ("quant_v", ctypes.c_int),
                ("p_range", ctypes.c_double), ("v_range", ctypes.c_double),
                ("sm_scale", ctypes.c_double), ("causal", ctypes.c_int)]


def _configure(lib):
    P = ctypes.c_void_p
    lib.oracle_e4m3_from_f32.argtypes = [ctypes.c_float]
    lib.oracle_e4m3_from_f32.restype = ctypes.c_uint8
    lib.oracle_e4m3_to_f64.argtypes = [ctypes.c_uint8]
    lib.oracle_e4m3_to_f64.restype = ctypes.c_double
    lib.oracle_int8_code.argtypes = [ctypes.c_float, ctypes.c_float]
    lib.oracle_int8_code.restype = ctypes.c_int8
    lib.oracle_int8_scale.argtypes = [ctypes.c_float]
    lib.oracle_int8_scale.restype = ctypes.c_float
    lib.oracle_f16_round.argtypes = [ctypes.c_float]
    lib.oracle_f16_round.restype = ctypes.c_double
    lib.oracle_prepass.argtypes = [ctypes.POINTER(_Cfg)] + [P] * 17
    lib.oracle_e2m1_from_f32.argtypes = [ctypes.c_float]
    lib.oracle_e2m1_from_f32.restype = ctypes.c_uint8
    lib.oracle_e2m1_to_f64.argtypes = [ctypes.c_uint8]
    lib.oracle_e2m1_to_f64.restype = ctypes.c_double
    lib.oracle_prepass.restype = ctypes.c_int
    lib.oracle_attn.argtypes = [ctypes.POINTER(_Cfg)] + [P] * 9 + [ctypes.c_int, P, P, P]
    lib.oracle_attn.restype = ctypes.c_int
    lib.oracle_ref_attn.argtypes = [ctypes.c_int] * 3 + [ctypes.c_double, ctypes.c_int, P, P, P, P]
    lib.oracle_ref_attn.restype = ctypes.c_int
    lib.oracle_num_threads.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            # SAGE_ORACLE_MUTATION selects a planted mistake, for the pins' own tests
            _lib = _configure(ctypes.CDLL(build(mutation=int(os.environ.get("SAGE_ORACLE_MUTATION", "0")))))
    return _lib


@contextlib.contextmanager
def mutant(mutation: int):
    """Run the oracle with planted mistake `mutation` inside the block (tests of the
    pins only)."""
    global _lib
    lib = _configure(ctypes.CDLL(build(mutation=mutation)))
    with _lock:
        saved, _lib = _lib, lib
    try:
        yield
    finally:
        with _lock:
            _lib = saved


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


# ---------------------------------------------------------------------------
# Codecs
# ---------------------------------------------------------------------------
def e4m3_encode(x) -> np.ndarray:
    """E4M3 (e4m3fn) code of each value, rounded to fp32 first; RNE, saturating to +-448.

    Pinned against torch.float8_e4m3fn on every value it does not saturate, and
    by decoding all 256 codes against the format's definition."""
    lib = _load()
    xs = np.asarray(x, dtype=np.float32).ravel()
    out = np.fromiter((lib.oracle_e4m3_from_f32(float(v)) for v in xs), dtype=np.uint8, count=xs.size)
    return out.reshape(np.shape(x))


def e4m3_decode(codes) -> np.ndarray:
    lib = _load()
    cs = np.asarray(codes, dtype=np.uint8).ravel()
    out = np.fromiter((lib.oracle_e4m3_to_f64(int(c)) for c in cs), dtype=np.float64, count=cs.size)
    return out.reshape(np.shape(codes))


def int8_code(xs, delta) -> np.ndarray:
    """INT8 code: round-half-even of the fp32 quotient xs / delta, clamped to +-127."""
    lib = _load()
    xs = np.asarray(xs, dtype=np.float32).ravel()
    ds = np.broadcast_to(np.asarray(delta, dtype=np.float32), xs.shape).ravel()
    return np.fromiter((lib.oracle_int8_code(float(a), float(b)) for a, b in zip(xs, ds)),
                       dtype=np.int8, count=xs.size)


def int8_scale(amax: float) -> float:
    return float(_load().oracle_int8_scale(float(amax)))


# ---------------------------------------------------------------------------
# Granularities (group sizes in rows of Q / keys of K); any divisor of 128 works.
# ---------------------------------------------------------------------------
GRANULARITY = {
    "per_block": (128, 128),
    "per_warp": (32, 128),
    "per_threadgroup": (32, 16),
}


def _cfg(n_q, n_kv, d, g_q, g_k, smooth_q, smooth_k, quant, p_range, v_range, sm_scale, causal):
    qqk, qp, qv = quant
    return _Cfg(n_q, n_kv, d, g_q, g_k, int(smooth_q), int(smooth_k), int(qqk), int(qp), int(qv),
                float(p_range), float(v_range), float(sm_scale), int(causal))


# quant = (QK, P, V): 1 = the method's INT8 / E4M3 / E4M3, 0 = exact.  PV_FP16 is the
# "qk_int8_pv_fp16" mode of the SageAttention deployment guide: P~ and V rounded to
# IEEE fp16 (P unscaled, V without per-channel scale), the PV product in fp16 x fp16.
PV_FP8 = (1, 1, 1)
PV_FP16 = (1, 2, 2)
# FP4 Q / K ("4+8": 4-bit QK^T, FP8 PV), in the microscaling form B200's tensor cores
# take: E2M1 codes, an E4M3 scale per 16 channels of each row and an fp32 scale per
# 128-row Q block / 128-key K tile (q_sf / k_sf hold the E4M3 scale codes).
QK_FP4_PV_FP8 = (2, 1, 1)


def e2m1_encode(x) -> np.ndarray:
    """E2M1 codes (round to nearest, ties to even mantissa, saturating at +-6)."""
    lib = _load()
    return np.array([lib.oracle_e2m1_from_f32(float(v)) for v in np.asarray(x, np.float32).ravel()],
                    np.uint8).reshape(np.shape(x))


def e2m1_decode(codes) -> np.ndarray:
    lib = _load()
    return np.array([lib.oracle_e2m1_to_f64(int(c)) for c in np.asarray(codes).ravel()]).reshape(np.shape(codes))


def f16_round(x):
    """IEEE fp16 rounding (ties to even) of fp32 values, as fp64 (the oracle's codec)."""
    lib = _load()
    return np.array([lib.oracle_f16_round(float(v)) for v in np.asarray(x, np.float32).ravel()]).reshape(np.shape(x))


def prepass_head(q, k, v, *, g_q=32, g_k=16, smooth_q=True, smooth_k=True,
                 quant=(1, 1, 1), p_range=448.0, v_range=448.0):
    """Smoothing + quantization of one head.  q: [Nq, d], k, v: [Nkv, d] (any float dtype,
    converted to fp64 exactly).  Returns a dict of the pre-pass tensors (see sage_oracle.c)."""
    lib = _load()
    q = np.ascontiguousarray(q, dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    nq, d = q.shape
    nk = k.shape[0]
    tq = -(-nq // TILE)
    nq_pad, nk_pad = tq * TILE, -(-nk // TILE) * TILE
    cfg = _cfg(nq, nk, d, g_q, g_k, smooth_q, smooth_k, quant, p_range, v_range, 1.0, 0)
    r = dict(
        qbar=np.zeros((tq, d), np.float32), kbar=np.zeros((d,), np.float32),
        q_code=np.zeros((nq_pad, d), np.int8), q_hat=np.zeros((nq_pad, d), np.float64),
        dq_row=np.zeros((nq_pad,), np.float32),
        k_code=np.zeros((nk_pad, d), np.int8), k_hat=np.zeros((nk_pad, d), np.float64),
        dk_key=np.zeros((nk_pad,), np.float32), k_s=np.zeros((max(nk, 1), d), np.float64),
        v_code=np.zeros((max(nk, 1), d), np.uint8), v_hat=np.zeros((max(nk, 1), d), np.float64),
        dv=np.zeros((d,), np.float32),
        q_sf=np.zeros((nq_pad, max(d // 16, 1)), np.uint8), k_sf=np.zeros((nk_pad, max(d // 16, 1)), np.uint8),
    )
    rc = lib.oracle_prepass(ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v),
                            _ptr(r["qbar"]), _ptr(r["kbar"]),
                            _ptr(r["q_code"]), _ptr(r["q_hat"]), _ptr(r["dq_row"]),
                            _ptr(r["k_code"]), _ptr(r["k_hat"]), _ptr(r["dk_key"]), _ptr(r["k_s"]),
                            _ptr(r["v_code"]), _ptr(r["v_hat"]), _ptr(r["dv"]), _ptr(r["q_sf"]), _ptr(r["k_sf"]))
    if rc != 0:
        raise ValueError("oracle_prepass failed with code %d" % rc)
    r["k_s"] = r["k_s"][:nk]
    r["v_code"] = r["v_code"][:nk]
    r["v_hat"] = r["v_hat"][:nk]
    r["cfg"] = dict(n_q=nq, n_kv=nk, d=d, g_q=g_q, g_k=g_k, smooth_q=smooth_q, smooth_k=smooth_k,
                    quant=tuple(quant), p_range=p_range, v_range=v_range)
    r["q"] = q
    return r


def delta_s(pre, t: int) -> np.ndarray:
    """Q-smoothing bias of Q block t over all keys: dS[t, j] = qbar_t . (K[j] - kbar), fp64."""
    return pre["k_s"] @ pre["qbar"][t].astype(np.float64)


def attn_head(pre, *, causal=False, sm_scale=None, qblocks=None, return_stats=False):
    """Attention of one head from ``prepass_head`` output.  Returns O [Nq, d] fp64; rows of
    Q blocks not listed in ``qblocks`` are left 0."""
    lib = _load()
    c = pre["cfg"]
    nq, nk, d = c["n_q"], c["n_kv"], c["d"]
    if sm_scale is None or sm_scale <= 0:
        sm_scale = 1.0 / np.sqrt(d)
    tq = -(-nq // TILE)
    blocks = np.arange(tq, dtype=np.int32) if qblocks is None else np.ascontiguousarray(qblocks, dtype=np.int32)
    cfg = _cfg(nq, nk, d, c["g_q"], c["g_k"], c["smooth_q"], c["smooth_k"], c["quant"],
               c["p_range"], c["v_range"], sm_scale, causal)
    o = np.zeros((max(nq, 1), d), np.float64)
    rl = np.zeros((max(nq, 1),), np.float64)
    rm = np.full((max(nq, 1),), -np.inf, np.float64)
    k_s = np.ascontiguousarray(pre["k_s"]) if nk > 0 else np.zeros((1, d))
    v_hat = np.ascontiguousarray(pre["v_hat"]) if nk > 0 else np.zeros((1, d))
    rc = lib.oracle_attn(ctypes.byref(cfg), _ptr(pre["qbar"]), _ptr(pre["q_hat"]), _ptr(pre["dq_row"]),
                         _ptr(pre["k_hat"]), _ptr(pre["dk_key"]), _ptr(k_s),
                         _ptr(v_hat), _ptr(pre["dv"]), _ptr(blocks), int(blocks.size),
                         _ptr(o), _ptr(rl), _ptr(rm))
    if rc != 0:
        raise ValueError("oracle_attn failed with code %d" % rc)
    o, rl, rm = o[:nq], rl[:nq], rm[:nq]
    if return_stats:
        return o, rl, rm
    return o


def lse_head(pre, *, causal=False, sm_scale=None, qblocks=None):
    """Log-sum-exp (natural log) of each row's attention logits, as the method computes
    them, referred back to the unsmoothed logits sm_scale * q_i . k_j.

    The method's logits are x_ij = sm_scale * S_ij with S = dQ dK S_int + qbar_t . K_s
    (steps of ``attn_head``).  K smoothing shifts every logit of row i by the same
    -sm_scale * q_i . kbar (q . K_s = q . K - q . kbar), which softmax ignores but the
    log-sum-exp does not; it is added back here so that the value approximates
    log sum_j exp(sm_scale q_i . k_j), the quantity that merges partial results over
    key ranges.  lse_i = m_i + log(l_i) + sm_scale q_i . kbar, with m, l the running max
    and sum of the online softmax; -inf for a row that sees no key.  Rows of Q blocks not
    in ``qblocks`` are -inf."""
    c = pre["cfg"]
    d = c["d"]
    if sm_scale is None or sm_scale <= 0:
        sm_scale = 1.0 / np.sqrt(d)
    _, rl, rm = attn_head(pre, causal=causal, sm_scale=sm_scale, qblocks=qblocks, return_stats=True)
    shift = sm_scale * (pre["q"] @ pre["kbar"].astype(np.float64))
    out = np.full(rl.shape, -np.inf)
    ok = rl > 0
    out[ok] = rm[ok] + np.log(rl[ok]) + shift[ok]
    return out


def _group(H: int, H_kv: int) -> int:
    """Query heads per key/value head."""
    if H_kv < 1 or H % H_kv != 0:
        raise ValueError("key/value heads (%d) must divide query heads (%d)" % (H_kv, H))
    return H // H_kv


def sage_attention(q, k, v, *, causal=False, sm_scale=None, granularity="per_threadgroup",
                   smooth_q=True, smooth_k=True, quant=(1, 1, 1), p_range=448.0, v_range=448.0,
                   heads=None, qblocks=None):
    """Whole quantized attention forward on [B, H, N, d] arrays (head-major).

    k and v may hold H_kv heads, H_kv dividing H (grouped-query attention): query head
    h reads key/value head h // (H // H_kv), and the method runs on that pair as on a
    multi-head pair.  ``heads``: optional list of (b, h) to compute (others stay 0);
    ``qblocks``: optional list of Q block indices to compute within each head.
    Returns O fp64 [B, H, Nq, d]."""
    q = np.asarray(q)
    k = np.asarray(k)
    v = np.asarray(v)
    B, H, nq, d = q.shape
    group = _group(H, k.shape[1])
    g_q, g_k = GRANULARITY[granularity] if isinstance(granularity, str) else granularity
    o = np.zeros((B, H, nq, d), np.float64)
    hs = [(b, h) for b in range(B) for h in range(H)] if heads is None else heads
    for b, h in hs:
        pre = prepass_head(q[b, h], k[b, h // group], v[b, h // group], g_q=g_q, g_k=g_k, smooth_q=smooth_q,
                           smooth_k=smooth_k, quant=quant, p_range=p_range, v_range=v_range)
        o[b, h] = attn_head(pre, causal=causal, sm_scale=sm_scale, qblocks=qblocks)
    return o


def sage_attention_varlen(q, k, v, cu_q, cu_kv, *, causal=False, sm_scale=None, return_lse=False, **kw):
    """Quantized attention of a packed batch: q [total_q, H, d], k, v [total_kv, H_kv, d]
    (token-major), sequence b holding tokens [cu_q[b], cu_q[b+1]) of q and
    [cu_kv[b], cu_kv[b+1]) of k and v.  Each sequence is attended on its own: the method
    runs on (q, k, v) of that sequence as on a batch of one (``sage_attention``
    arguments in ``kw``); causal is bottom-right aligned per sequence.  Returns O
    [total_q, H, d] fp64 (tokens no sequence covers stay 0) and, with return_lse, the
    rows' log-sum-exp [total_q, H] (``lse_head``)."""
    q = np.asarray(q)
    k = np.asarray(k)
    v = np.asarray(v)
    total_q, H, d = q.shape
    group = _group(H, k.shape[1])
    g_q, g_k = GRANULARITY[kw.pop("granularity", "per_threadgroup")]
    o = np.zeros((total_q, H, d), np.float64)
    lse = np.full((total_q, H), -np.inf)
    for b in range(len(cu_q) - 1):
        q0, q1, k0, k1 = int(cu_q[b]), int(cu_q[b + 1]), int(cu_kv[b]), int(cu_kv[b + 1])
        if q1 <= q0:
            continue
        for h in range(H):
            pre = prepass_head(q[q0:q1, h], k[k0:k1, h // group], v[k0:k1, h // group], g_q=g_q, g_k=g_k, **kw)
            o[q0:q1, h] = attn_head(pre, causal=causal, sm_scale=sm_scale)
            if return_lse:
                lse[q0:q1, h] = lse_head(pre, causal=causal, sm_scale=sm_scale)
    return (o, lse) if return_lse else o


def reference_attention(q, k, v, *, causal=False, sm_scale=None, heads=None):
    """Textbook full-precision attention in fp64 (two-pass softmax), [B, H, N, d].
    k and v may hold fewer heads than q, as in sage_attention."""
    lib = _load()
    q = np.asarray(q)
    B, H, nq, d = q.shape
    nk = np.asarray(k).shape[2]
    group = _group(H, np.asarray(k).shape[1])
    if sm_scale is None or sm_scale <= 0:
        sm_scale = 1.0 / np.sqrt(d)
    o = np.zeros((B, H, nq, d), np.float64)
    hs = [(b, h) for b in range(B) for h in range(H)] if heads is None else heads
    for b, h in hs:
        qq = np.ascontiguousarray(q[b, h], dtype=np.float64)
        kk = np.ascontiguousarray(np.asarray(k)[b, h // group], dtype=np.float64)
        vv = np.ascontiguousarray(np.asarray(v)[b, h // group], dtype=np.float64)
        oo = np.zeros((max(nq, 1), d), np.float64)
        lib.oracle_ref_attn(nq, nk, d, float(sm_scale), int(causal), _ptr(qq), _ptr(kk), _ptr(vv), _ptr(oo))
        o[b, h] = oo[:nq]
    return o
