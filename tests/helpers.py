"""Shared helpers of the GPU parity tests: run the CUDA path and the oracle on the
same seeded inputs and compare."""
import math

import numpy as np
import torch

import oracle
import quantized_attention_fine_b200 as sage

# Tolerances of the attention output against the oracle (fp64) and against
# full-precision attention.
O_MAX_ABS = 1e-2
O_COS_ORACLE = 0.9999
O_COS_FULL = 0.995

GRAN_OF = {"per_block": (128, 128), "per_warp": (32, 128), "per_threadgroup": (32, 16)}


def cos(a, b) -> float:
    a = np.asarray(a, dtype=np.float64).ravel()
    b = np.asarray(b, dtype=np.float64).ravel()
    den = math.sqrt(float((a * a).sum()) * float((b * b).sum()))
    return float((a * b).sum() / den) if den > 0 else (1.0 if np.array_equal(a, b) else 0.0)


def to_np64(x: torch.Tensor) -> np.ndarray:
    return x.detach().to("cpu").double().numpy()


def head_slices(q, k, v, b, h, layout):
    """[N, d] slices of one head from HND or NHD tensors (CPU)."""
    if layout == "HND":
        return q[b, h], k[b, h], v[b, h]
    return q[b, :, h], k[b, :, h], v[b, :, h]


def oracle_head(qh, kh, vh, *, causal, granularity="per_threadgroup", smooth_q=True, smooth_k=True,
                p_range=448.0, v_range=448.0, qblocks=None, sm_scale=None):
    g_q, g_k = GRAN_OF[granularity]
    pre = oracle.prepass_head(to_np64(qh), to_np64(kh), to_np64(vh), g_q=g_q, g_k=g_k, smooth_q=smooth_q,
                              smooth_k=smooth_k, p_range=p_range, v_range=v_range)
    o = oracle.attn_head(pre, causal=causal, qblocks=qblocks, sm_scale=sm_scale)
    return pre, o


def rows_of_blocks(n_q, qblocks):
    rows = []
    for t in qblocks:
        rows.extend(range(t * 128, min(t * 128 + 128, n_q)))
    return np.asarray(rows, dtype=np.int64)


def assert_close_to_oracle(o_gpu, o_orc, what=""):
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    err = np.max(np.abs(o_gpu - o_orc)) if o_gpu.size else 0.0
    c = cos(o_gpu, o_orc)
    assert err <= O_MAX_ABS, "%s: max |O_gpu - O_oracle| = %.3e > %.0e" % (what, err, O_MAX_ABS)
    assert c >= O_COS_ORACLE, "%s: cos(O_gpu, O_oracle) = %.6f < %.4f" % (what, c, O_COS_ORACLE)
    return err, c


def storage_positions(n_pad: int) -> np.ndarray:
    """Position of key j in the workspace's key-ordered arrays (V^T codes, dS): inside
    each 128-key tile the tile's even keys come first, then its odd keys."""
    j = np.arange(n_pad)
    k = j % 128
    return (j - k) + (k & 1) * 64 + (k >> 1)


def natural_key_order(x: np.ndarray) -> np.ndarray:
    """An array whose last axis is in the workspace's key storage order -> natural key order."""
    return x[..., storage_positions(x.shape[-1])]

