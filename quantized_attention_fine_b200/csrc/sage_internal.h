// sage_internal.h -- host-side shared definitions of libsage_b200: workspace
// layout, kernel parameter blocks and launcher prototypes.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/sage.h"

namespace sage {

constexpr int kTile = 128;        // Q block rows = KV tile keys (part of the numerics)
constexpr int kKeyRun = 16;       // delta_K is stored once per 16 keys
constexpr int kStatChunk = 512;   // tokens per CTA of the K-mean / V-amax pass
constexpr size_t kWsAlign = 1024;
constexpr size_t kStatusBytes = 256;

// H query heads share H_kv key/value heads (H_kv divides H; H_kv = H is multi-head
// attention): query head h reads key/value head h / (H / H_kv).
// Variable-length batches (varlen = 1): B sequences packed token-major, sequence b
// holding tokens [cu[b], cu[b + 1]) of [total][heads][d] tensors; n_q and n_kv are then
// the longest lengths, and every per-sequence workspace array is padded to them.
struct Shape {
    int B, H, H_kv, n_q, n_kv, d;
    int BH, BH_kv, Tq, Tk, nq_pad, nk_pad, n_chunks;
    int varlen, total_q, total_kv;
    int pv16;   // FP16 P / V mode: the transposed V holds 2 bytes per element
    int fp4;    // FP4 Q / K mode: E2M1 codes and E4M3 scale atoms (sfq, sfk regions)
};

inline Shape make_shape(int B, int H, int H_kv, int n_q, int n_kv, int d) {
    Shape s;
    s.B = B; s.H = H; s.H_kv = H_kv; s.n_q = n_q; s.n_kv = n_kv; s.d = d;
    s.varlen = 0; s.total_q = 0; s.total_kv = 0; s.pv16 = 0; s.fp4 = 0;
    s.BH = B * H;
    s.BH_kv = B * H_kv;
    s.Tq = (n_q + kTile - 1) / kTile;
    s.Tk = (n_kv + kTile - 1) / kTile;
    s.nq_pad = s.Tq * kTile;
    s.nk_pad = s.Tk * kTile;
    s.n_chunks = (n_kv + kStatChunk - 1) / kStatChunk;
    if (s.n_chunks < 1) s.n_chunks = 1;
    return s;
}

// Byte offsets of every workspace region.
struct WsLayout {
    size_t status, q8, k8, vt8, dq, dk, dv, qbar, kbar, ds, qs_kbar, lse, ksum_part, vmax_part, sfq, sfk, total;
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline WsLayout ws_layout(const Shape &s) {
    WsLayout w;
    const size_t BH = (size_t)s.BH, BHk = (size_t)s.BH_kv, d = (size_t)s.d;
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes, kWsAlign); return o; };
    w.status = take(kStatusBytes);
    w.q8 = take(BH * s.nq_pad * d);
    w.k8 = take(BHk * s.nk_pad * d);
    w.vt8 = take(BHk * d * s.nk_pad * (s.pv16 ? 2 : 1));
    w.dq = take(BH * s.nq_pad * 4);
    w.dk = take(BHk * (s.nk_pad / kKeyRun) * 4);
    w.dv = take(BHk * d * 4);
    w.qbar = take(BH * s.Tq * d * 4);
    w.kbar = take(BHk * d * 4);
    w.ds = take(BH * s.Tq * (size_t)s.nk_pad * 4);
    w.qs_kbar = take(BH * s.nq_pad * 4);
    w.lse = take(BH * s.nq_pad * 4);
    w.ksum_part = take(BHk * s.n_chunks * d * 8);
    w.vmax_part = take(BHk * s.n_chunks * d * 4);
    // FP4 scale atoms: 512 bytes per 128-row tile and 64-channel chunk
    w.sfq = take(s.fp4 ? BH * s.Tq * (d / 64) * 512 : 0);
    w.sfk = take(s.fp4 ? BHk * s.Tk * (d / 64) * 512 : 0);
    w.total = off;
    return w;
}

// Token offset and length of sequence b of a packed batch (cu: B + 1 offsets), clamped
// so that the range lies inside [0, total) and is no longer than n_max.  Without cu
// (a dense batch) every sequence has length n_max and the offset is unused.
struct SeqRange {
    int off, n;
};
__host__ __device__ __forceinline__ SeqRange seq_range(const int *cu, int b, int n_max, int total) {
    if (!cu) return SeqRange{0, n_max};
    int a0 = cu[b], a1 = cu[b + 1];
    a0 = a0 < 0 ? 0 : (a0 > total ? total : a0);
    a1 = a1 < a0 ? a0 : (a1 > total ? total : a1);
    const int n = a1 - a0;
    return SeqRange{a0, n < n_max ? n : n_max};
}

// Element strides of a [B, H, N, d] (HND) or [B, N, H, d] (NHD) tensor.
struct Strides {
    int64_t b, h, n;
};
inline Strides make_strides(int layout, int H, int N, int d) {
    Strides st;
    if (layout == 0) { st.b = (int64_t)H * N * d; st.h = (int64_t)N * d; st.n = d; }
    else { st.b = (int64_t)N * H * d; st.h = d; st.n = (int64_t)H * d; }
    return st;
}

struct PrepassArgs {
    // tensor maps of the caller's 16-bit Q, K, V ([BH][n][d] or [B][n][H][d]; d x 128-row
    // boxes, no swizzle), valid where the pointer below is not null
    CUtensorMap tm_q, tm_k, tm_v;
    // store map of the V^T codes (the workspace's [BH_kv * d][nk_pad] bytes, 128-key x
    // d boxes, 128-byte swizzle), valid where v is not null and V is quantized to E4M3
    CUtensorMap tm_vt;
    const void *q, *k, *v;   // any may be null: that part is skipped
    int bf16, nhd;
    const int *cu_q, *cu_kv;  // packed batch offsets (device), or null for a dense batch
    Strides sq, skv;
    Shape shape;
    int g_q, g_k, smooth_q, smooth_k;
    float v_range;
    int pv16;   // FP16 V (no per-channel scale: delta_V = 1) instead of E4M3 codes
    int fp4;    // FP4 Q / K (E2M1 codes, E4M3 block scales, per-tile fp32 scales)
    uint8_t *ws;
    WsLayout L;
};

struct AttnParams {
    const float *dq, *dk, *dv, *ds;
    const float *qs_kbar;   // per row: (q_i - qbar_t) . kbar, the logit shift of K smoothing
    float *lse;             // per row: log-sum-exp of the logits (natural log)
    void *o;
    int64_t so_b, so_h, so_n;
    int H, n_q, n_kv, Tq, Tk, nq_pad, nk_pad, BH;
    const int *cu_q, *cu_kv;  // packed batch offsets (device), or null for a dense batch
    int total_q, total_kv;
    int group;          // query heads per key/value head (H / H_kv)
    int H_kv;
    int head_block;     // query heads per block of the CTA order (set by launch_attention)
    int causal;
    int use_ds;         // 0: Q smoothing off, dS not read
    int pv16;           // FP16 P~ and V, kind::f16 PV (log2_pr is then 0)
    int fp4;            // FP4 Q / K, QK^T on kind::mxf4nvf4 (d = 64)
    const uint8_t *sfq, *sfk;   // FP4 scale atoms
    int out_bf16;
    float scale_log2;   // sm_scale * log2(e)
    float log2_pr;      // log2(Pr)
    int *status;
    int fault_inject;
    // Q quantized inside the attention kernel (fused_q): the kernel reads the caller's
    // 16-bit Q through its Q tensor map and 16-bit K through the raw-K map, forms
    // qbar, delta_Q and the INT8 codes of its own Q tiles and the dS rows of every key
    // tile; dq / ds / qs_kbar above are then unused.
    int fused_q;
    int g_q;                 // rows per delta_Q group (32 or 128)
    int nhd;                 // token-major caller tensors (coordinates of the raw maps)
    const float *kbar;       // [BH_kv][d] K channel means
    float *qbar_w;           // [BH][Tq][d] written: qbar of every Q tile
    float *dq_w;             // [BH][nq_pad] written: delta_Q of every row
    int8_t *q8_dump;         // [BH][nq_pad][d] written when not null: the Q codes
};

cudaError_t launch_prepass(const PrepassArgs &a, cudaStream_t stream);
// dS = qbar . K^T on the tensor core.  tm_k: tensor map of the caller's 16-bit K
// (3-D [BH][n_kv][d] for head-major, 4-D [B][n_kv][H][d] for token-major, 64 x 128
// boxes, 128-byte swizzle; for a packed batch 4-D [1][total_kv][H_kv][d]).
// causal_skip: leave entries of Q blocks that can never see a key tile unwritten (key
// j visible to query i iff j <= i + causal_off; for a packed batch the offset is each
// sequence's n_kv - n_q and causal_off is unused).  cu_q, cu_kv: packed batch offsets
// or null.
cudaError_t launch_ds_gemm(const CUtensorMap &tm_k, float *ds_out, const float *qbar, const Shape &s,
                           int nhd, int bf16, int causal_skip, int causal_off, const int *cu_q, const int *cu_kv,
                           int *status, cudaStream_t stream);
// tq: Q codes, or with p.fused_q the caller's 16-bit Q (64-element x 128-row boxes,
// 128-byte swizzle); tkr: with p.fused_q the caller's 16-bit K (64-element x 16-key
// boxes, 128-byte swizzle), else unused.
cudaError_t launch_attention(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                             const CUtensorMap &tkr, const AttnParams &p, int d, cudaStream_t stream);
cudaError_t launch_debug_qk_tile(const CUtensorMap &tq, const CUtensorMap &tk, int d, int q_row0, int k_row0,
                                 int32_t *s_out, int *status, cudaStream_t stream);
cudaError_t launch_debug_pv(const uint8_t *p, const uint8_t *vt, int n_tiles, int d, float *o, int *status,
                            cudaStream_t stream, int acc_f16);
// n_ctas CTAs each issue n_iter tcgen05.mma of one kind (M = 128, N = 256) from
// shared memory into one tensor-memory accumulator; see sage_debug_mma_rate.
cudaError_t launch_debug_mma_rate(int kind, int n_iter, int n_ctas, int *status, cudaStream_t stream);
// FP4 (E2M1) quantization of fp32 rows [n_rows][d] with two-level scales, per 128-row
// tile; see sage_debug_quant_fp4.
cudaError_t launch_debug_quotient_check(const float *deltas, int n_delta, int bf16, unsigned long long *count,
                                        unsigned int *first, cudaStream_t stream);
cudaError_t launch_debug_quant_fp4(const float *xs, int n_rows, int d, uint8_t *codes, uint8_t *sf, float *g,
                                   cudaStream_t stream);
cudaError_t launch_zero_output(void *o, size_t bytes, cudaStream_t stream);
// One FP4 QK^T tile on the block-scaled tensor core; see sage_debug_qk_tile_fp4.
cudaError_t launch_debug_qk_fp4(const uint8_t *q4, const uint8_t *k4, const uint8_t *sfq, const uint8_t *sfk, int d,
                                float *out, int *status, cudaStream_t stream);

// How a whole-forward call (sage_attn_fwd_gqa's arguments) proceeds once its
// arguments are valid: nothing to do (B * H == 0 or n_q == 0), O = 0 without a
// workspace (n_kv == 0), or the full path with a workspace of *ws_need bytes.
enum FwdPlan { kFwdNoop = 0, kFwdZeroOut = 1, kFwdRun = 2 };
// Every check sage_attn_fwd_gqa makes before it enqueues anything, in the same order
// and with the same status; on SAGE_OK also the plan and the workspace size.
sage_status_t check_fwd_args(const void *q, const void *k, const void *v, const void *o, int dtype, int layout,
                             int B, int H, int H_kv, int n_q, int n_kv, int d, const sage_quant_mode_t *mode,
                             int *plan, size_t *ws_need);
// The scratch array of sage_attn_fwd_noalloc on the current device, 1024-byte
// aligned, and its usable bytes (the first call on a device looks its address up).
sage_status_t noalloc_workspace(uint8_t **ws, size_t *bytes);

}  // namespace sage
