/*
 * sage.h -- C ABI of libsage_b200.so: the smoothed-INT8-QK / FP8-PV quantized
 * attention forward (the SageAttention2 / SageAttention2++ method) on NVIDIA
 * B200 (sm_100a).
 *
 * What is computed (per batch b, head h; Q [N_q, d], K and V [N_kv, d]):
 *   1. K smoothing: K_s = K - mean over the N_kv valid tokens of K.
 *      ("SageAttention2" arXiv 2411.10958, abstract: outlier smoothing;
 *       zhaifeiyue.github.io notes on 2411.10958: fine-grained quantization + smoothing.)
 *   2. Q smoothing: for each 128-row Q block t, qbar_t = mean of its valid rows,
 *      Q_s = Q - qbar_t, and the bias dS[t, j] = qbar_t . K[j] is added back to the
 *      scores.  (2411.10958 abstract: "a method to smooth Q".)  Using K instead of
 *      K_s in dS changes every score of a row by the same constant, which softmax
 *      ignores.
 *   3. INT8 quantization of Q_s and K_s per group (g_q consecutive rows of a Q
 *      block, g_k consecutive keys of a 128-key tile): delta = amax / 127 (fp32),
 *      code = clamp(round-half-even(x / delta), -127, 127).
 *   4. V per channel: delta_V[c] = max_j |V[j, c]| / Vr, V8 = E4M3(V / delta_V).
 *      (pith.science verdict on arXiv 2505.21136, key_machinery.)
 *   5. S = delta_Q(i) delta_K(j) (Q_int . K_int) + dS, computed as an exact INT32
 *      tensor-core product; tiled online softmax over 128-key tiles with an exact
 *      rescale whenever a row maximum grows; P~ = exp(x - m) scaled by Pr and rounded
 *      to E4M3 (static scale 1 / Pr, since P~ <= 1); O += P8 . V8 on FP8 tensor cores
 *      with FP32 accumulation in tensor memory.
 *   6. O = acc / Pr * delta_V[c] / l, with l the sum of the unquantized P~; a row
 *      that sees no key is 0.  Rounded to the input dtype (round to nearest even).
 *   7. The row log-sum-exp of the logits, written to the workspace (SAGE_WS_LSE).
 * The FP16 P / V mode (sage_quant_mode_t.pv_fp16) replaces steps 4-6's E4M3 P and V
 * by fp16 P~ and V (no Pr, no delta_V) and the FP8 PV product by an FP16 one.
 *
 * Conventions for every entry point:
 *   - Device pointers are plain CUDA device addresses; `stream` is a cudaStream_t
 *     (NULL = legacy default stream).  All work is enqueued on `stream`; nothing
 *     synchronizes except sage_get_device_status.
 *   - Tensors: dtype SAGE_DTYPE_F16 / SAGE_DTYPE_BF16; layout SAGE_LAYOUT_HND is a
 *     contiguous [B, H, N, d] array, SAGE_LAYOUT_NHD a contiguous [B, N, H, d] array.
 *     Q, K, V and O share dtype and layout.  Base addresses must be 16-byte aligned.
 *   - d is 64 or 128.  The entry points without a suffix are multi-head (H query
 *     heads, H key/value heads).  The `_gqa` entry points take H query heads and
 *     H_kv key/value heads (H_kv divides H, grouped-query attention): query head h
 *     of batch b attends to key/value head h / (H / H_kv) of batch b.  K and V are
 *     then [B, H_kv, N_kv, d] (HND) or [B, N_kv, H_kv, d] (NHD); Q and O keep H.
 *     K smoothing and delta_V are properties of one key/value head and are shared
 *     by its query heads; Q smoothing and dS stay per query head.  (The pages
 *     validate the method on multi-head attention only and name grouped-query
 *     attention as a variant an attention backend must serve: notes on 2505.21136,
 *     the comparison with SGLang and the list of unvalidated variants.)
 *   - The caller owns all memory, including the workspace; the library allocates
 *     nothing and keeps no state between calls.  The workspace must be at least
 *     sage_workspace_bytes_mode(...) bytes for the mode used (sage_workspace_bytes
 *     for the default mode), 1024-byte aligned, and its first 256 bytes (the
 *     device status block) must be zero before first use.  Each entry point
 *     enqueues its launches on `stream` only and takes its parameters by value, so
 *     a call may be captured in a CUDA graph and replayed.
 *   - Argument errors return a status synchronously and enqueue nothing.  A launch
 *     failure returns SAGE_ERR_CUDA.  A device-side wait that runs out (about one
 *     second) makes the kernel stop early and record SAGE_ERR_TIMEOUT in the status
 *     block, read with sage_get_device_status.
 *   - B * H == 0 or N_q == 0 is a no-op returning SAGE_OK.  N_kv == 0 writes O = 0.
 */
#ifndef SAGE_B200_H
#define SAGE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(_WIN32)
#define SAGE_API
#else
#define SAGE_API __attribute__((visibility("default")))
#endif

typedef enum {
    SAGE_OK = 0,
    SAGE_ERR_INVALID_ARG = 1,  /* null pointer, bad size or enum                  */
    SAGE_ERR_UNSUPPORTED = 2,  /* valid but not supported: d, alignment, size cap  */
    SAGE_ERR_WORKSPACE = 3,    /* workspace smaller than sage_workspace_bytes      */
    SAGE_ERR_CUDA = 4,         /* a CUDA runtime / driver call failed              */
    SAGE_ERR_TIMEOUT = 5       /* a device-side bounded wait ran out               */
} sage_status_t;

typedef enum { SAGE_LAYOUT_HND = 0, SAGE_LAYOUT_NHD = 1 } sage_layout_t;
typedef enum { SAGE_DTYPE_F16 = 0, SAGE_DTYPE_BF16 = 1 } sage_dtype_t;

/* INT8 group sizes (g_q rows of Q, g_k keys of K).  The pages name the
 * granularities per block (SageAttention, "INT8 per-block") and per thread
 * (SageAttention2, thread-level); tcgen05 has no per-thread operand fragments, so
 * the finest mode groups 32 rows (one tensor-memory lane quadrant) and 16 keys. */
typedef enum {
    SAGE_QK_PER_BLOCK = 0,        /* g_q = 128, g_k = 128 */
    SAGE_QK_PER_WARP = 1,         /* g_q = 32,  g_k = 128 */
    SAGE_QK_PER_THREADGROUP = 2,  /* g_q = 32,  g_k = 16  (default) */
    SAGE_QK_FP4 = 3               /* 4-bit Q and K instead of INT8 (the pages' "4+8"
                                   * variant), in the block-scaled form B200's tensor
                                   * cores take: per 128-row tile an fp32 scale
                                   * g = amax / 2688 (1 if amax = 0); per row and 16
                                   * channels an E4M3 scale sf = E4M3(amax / g / 6) (1 if
                                   * that amax is 0, 2^-9 if it rounds to 0); per element
                                   * the E2M1 code of x / (g sf) (round to nearest even,
                                   * saturating at 6).  QK^T runs on tcgen05.mma
                                   * kind::mxf4nvf4.  The quantization calls take d = 64 or
                                   * 128; attention in this mode takes d = 64 (at d = 128
                                   * the four FP32 tensor-memory accumulators of the two Q
                                   * tiles fill all 512 columns and leave none for the
                                   * scales: SAGE_ERR_UNSUPPORTED).  FP8 P / V only. */
} sage_qk_gran_t;

typedef struct {
    int32_t gran;      /* sage_qk_gran_t                                        */
    int32_t smooth_q;  /* 1: subtract per-block Q mean and add dS back          */
    int32_t smooth_k;  /* 1: subtract per-head K mean                           */
    float p_range;     /* Pr, (0, 448]; 448 = full E4M3 range (default)         */
    float v_range;     /* Vr, (0, 448]; 448 (SageAttention2 default)            */
    int32_t pv_fp16;   /* 0: E4M3 P (x Pr) and per-channel E4M3 V, FP8 PV (default);
                        * 1: FP16 P~ (unscaled) and FP16 V (no per-channel scale),
                        *    FP16 PV with FP32 accumulation: the deployment guide's
                        *    "qk_int8_pv_fp16" high-fidelity mode; p_range and v_range
                        *    are unused.  The workspace of this mode is larger
                        *    (sage_workspace_bytes_mode). */
} sage_quant_mode_t;
/* A NULL mode pointer means {SAGE_QK_PER_THREADGROUP, 1, 1, 448, 448, 0}.
 * In the SAGE_QK_FP4 mode the workspace views change as follows: SAGE_WS_Q8 / SAGE_WS_K8
 * hold the E2M1 codes, [rows][d/2] bytes (channel 2c in the low nibble of byte c) in the
 * same regions; SAGE_WS_DQ holds each row's tile scale g, SAGE_WS_DK each 16-key run's
 * tile scale g; SAGE_WS_SFQ / SAGE_WS_SFK hold the E4M3 scales per 128-row tile and
 * 64-channel chunk as 512-byte atoms (the scale of tile row m and block b at byte
 * 16 (m mod 32) + 4 (m / 32) + (b mod 4) of atom b / 4): [BH][Tq][d/64][512] and
 * [BHk][Tk][d/64][512]. */

/* Bytes of workspace for one problem size (any dtype/layout).  0 on bad sizes. */
SAGE_API size_t sage_workspace_bytes(int B, int H, int n_q, int n_kv, int d);
SAGE_API size_t sage_workspace_bytes_gqa(int B, int H, int H_kv, int n_q, int n_kv, int d);
/* Bytes of workspace for a mode (NULL = default): the FP16 P / V mode needs 2 bytes per
 * V element instead of 1; every other mode field leaves the size unchanged. */
SAGE_API size_t sage_workspace_bytes_mode(int B, int H, int H_kv, int n_q, int n_kv, int d,
                                          const sage_quant_mode_t *mode);

/* Steps 1-3 (and the dS bias) for Q and K into the workspace.
 * q: [B,H,n_q,d] or [B,n_q,H,d]; k: [B,H,n_kv,d] or [B,n_kv,H,d]. */
SAGE_API sage_status_t sage_quant_qk(const void *q, const void *k, int dtype, int layout,
                                     int B, int H, int n_q, int n_kv, int d,
                                     const sage_quant_mode_t *mode,
                                     void *workspace, size_t workspace_bytes, void *stream);
SAGE_API sage_status_t sage_quant_qk_gqa(const void *q, const void *k, int dtype, int layout,
                                         int B, int H, int H_kv, int n_q, int n_kv, int d,
                                         const sage_quant_mode_t *mode,
                                         void *workspace, size_t workspace_bytes, void *stream);

/* Step 4 for V into the workspace (n_q only sizes the workspace regions). */
SAGE_API sage_status_t sage_quant_v(const void *v, int dtype, int layout,
                                    int B, int H, int n_q, int n_kv, int d,
                                    const sage_quant_mode_t *mode,
                                    void *workspace, size_t workspace_bytes, void *stream);
SAGE_API sage_status_t sage_quant_v_gqa(const void *v, int dtype, int layout,
                                        int B, int H, int H_kv, int n_q, int n_kv, int d,
                                        const sage_quant_mode_t *mode,
                                        void *workspace, size_t workspace_bytes, void *stream);

/* Steps 5-6 from a workspace filled by sage_quant_qk and sage_quant_v with the same
 * sizes and mode.  o: output, same dtype/layout as the inputs were.
 * sm_scale <= 0 means 1/sqrt(d).  causal: key j is visible to query i iff
 * j <= i + n_kv - n_q (bottom-right aligned). */
SAGE_API sage_status_t sage_attn_fwd_prequant(void *o, int dtype, int layout,
                                              int B, int H, int n_q, int n_kv, int d,
                                              int causal, float sm_scale,
                                              const sage_quant_mode_t *mode,
                                              const void *workspace, size_t workspace_bytes,
                                              void *stream);
SAGE_API sage_status_t sage_attn_fwd_prequant_gqa(void *o, int dtype, int layout,
                                                  int B, int H, int H_kv, int n_q, int n_kv, int d,
                                                  int causal, float sm_scale,
                                                  const sage_quant_mode_t *mode,
                                                  const void *workspace, size_t workspace_bytes,
                                                  void *stream);

/* The whole forward: quant_qk + quant_v + attn_fwd_prequant, enqueued on `stream`. */
SAGE_API sage_status_t sage_attn_fwd(const void *q, const void *k, const void *v, void *o,
                                     int dtype, int layout, int B, int H, int n_q, int n_kv,
                                     int d, int causal, float sm_scale,
                                     const sage_quant_mode_t *mode,
                                     void *workspace, size_t workspace_bytes, void *stream);
SAGE_API sage_status_t sage_attn_fwd_gqa(const void *q, const void *k, const void *v, void *o,
                                         int dtype, int layout, int B, int H, int H_kv, int n_q,
                                         int n_kv, int d, int causal, float sm_scale,
                                         const sage_quant_mode_t *mode,
                                         void *workspace, size_t workspace_bytes, void *stream);

/* The whole forward with Q quantized inside the attention kernel ("SageAttention2"
 * abstract: Q is smoothed per 128-row block, so a block's mean, delta_Q and codes need
 * only that block):
 *   K / V pre-pass (K mean, K codes, delta_V, V codes)  ->  attention
 * where the attention kernel reads the caller's 16-bit Q tiles, smooths and quantizes
 * them (codes, delta_Q and qbar bit-identical to sage_quant_qk's), and forms the dS
 * bias qbar . K of every key tile from the caller's K on one of its warps.  The
 * results equal sage_attn_fwd_gqa's up to the rounding of dS (its products are summed
 * in another order).  On B200 this path is slower than sage_attn_fwd_gqa (the dS
 * warp reads every key tile's 16-bit K again and its products run on the warp-level
 * tensor-core path); it is kept as an alternative, not the default.
 * With v == NULL only the attention runs, on a workspace whose K / V parts were
 * filled for the same sizes and mode (by sage_quant_qk + sage_quant_v, or by an
 * earlier call).  The workspace then holds qbar (SAGE_WS_QBAR) and delta_Q
 * (SAGE_WS_DQ) of the call; SAGE_WS_Q8, SAGE_WS_DS and SAGE_WS_QS_KBAR are not
 * written (the Q codes are, under sage_debug_set_q_code_dump).  Arguments and errors
 * as sage_attn_fwd_gqa; SAGE_ERR_UNSUPPORTED for the 4-bit mode (SAGE_QK_FP4), whose
 * Q is quantized in the pre-pass. */
SAGE_API sage_status_t sage_attn_fwd_qfused_gqa(const void *q, const void *k, const void *v, void *o, int dtype,
                                                int layout, int B, int H, int H_kv, int n_q, int n_kv, int d,
                                                int causal, float sm_scale, const sage_quant_mode_t *mode,
                                                void *workspace, size_t workspace_bytes, void *stream);

/* Diagnostic switch (process-wide, not for concurrent use): while enabled (1), forward
 * calls that quantize Q inside the attention kernel also write the Q codes to the
 * workspace's SAGE_WS_Q8 view, so that they can be compared with sage_quant_qk's.
 * 0 disables (the default).  SAGE_ERR_INVALID_ARG for other values. */
SAGE_API sage_status_t sage_debug_set_q_code_dump(int enable);

/* ---- variable-length (packed) batches -------------------------------------------
 * B sequences of different lengths packed token-major, as in the pages' varlen
 * kernels (the deployment guide's "dynamic sequence length" tip: a per-block causal
 * varlen attention):
 *   q, o : [total_q,  H,    d], sequence b holding tokens [cu_seqlens_q[b], cu_seqlens_q[b+1])
 *   k, v : [total_kv, H_kv, d], sequence b holding tokens [cu_seqlens_kv[b], cu_seqlens_kv[b+1])
 * cu_seqlens_q / cu_seqlens_kv: DEVICE int32 arrays of B + 1 nondecreasing offsets
 * starting at 0 and ending at most at total_q / total_kv.  Each sequence is attended on
 * its own, with the method's steps per sequence and head (K mean, delta_V, Q blocks of
 * 128 rows, causal bottom-right aligned per sequence: key j visible to query i iff
 * j <= i + n_kv,b - n_q,b).  max_seqlen_q / max_seqlen_kv must be at least every
 * sequence's length (longer sequences are cut to them); the workspace is sized by them
 * (sage_workspace_bytes_varlen), its per-sequence arrays padded to these lengths and
 * indexed as for a dense batch of B sequences (the SAGE_WS_* views below, with
 * n_q = max_seqlen_q, n_kv = max_seqlen_kv).  Work scales with the actual lengths:
 * tiles past a sequence's end are skipped.  Offsets outside [0, total] are clamped;
 * tokens of o that no sequence covers are not written.  total_kv == 0 writes o = 0.
 * Other arguments and errors as sage_attn_fwd_gqa. */
SAGE_API size_t sage_workspace_bytes_varlen(int B, int H, int H_kv, int max_seqlen_q, int max_seqlen_kv, int d);
SAGE_API sage_status_t sage_attn_fwd_varlen(const void *q, const void *k, const void *v, void *o, int dtype,
                                            const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_kv,
                                            int B, int H, int H_kv, int total_q, int total_kv,
                                            int max_seqlen_q, int max_seqlen_kv, int d, int causal,
                                            float sm_scale, const sage_quant_mode_t *mode,
                                            void *workspace, size_t workspace_bytes, void *stream);
/* The same with Q quantized inside the attention kernel (as sage_attn_fwd_qfused_gqa). */
SAGE_API sage_status_t sage_attn_fwd_varlen_qfused(const void *q, const void *k, const void *v, void *o, int dtype,
                                                   const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_kv,
                                                   int B, int H, int H_kv, int total_q, int total_kv,
                                                   int max_seqlen_q, int max_seqlen_kv, int d, int causal,
                                                   float sm_scale, const sage_quant_mode_t *mode,
                                                   void *workspace, size_t workspace_bytes, void *stream);

/* The whole forward, exactly as sage_attn_fwd, for callers that must not allocate
 * device memory (for example a plugin whose host application owns every device
 * allocation, or a serving loop where a cudaMalloc, which can synchronize the
 * device, is not acceptable) and so cannot provide a workspace.  The pages have no
 * counterpart of this entry point.
 *   - Scratch: one 64 MiB device array inside the library, held on every GPU where
 *     the library's device code is loaded, until the process exits.  Problems whose
 *     sage_workspace_bytes_mode(B, H, H, n_q, n_kv, d, mode) exceeds 64 MiB - 1 KiB
 *     are refused with SAGE_ERR_WORKSPACE before anything is enqueued.
 *   - Allocates nothing itself: no cudaMalloc / cudaFree or allocating library call.
 *     Under CUDA's default lazy module loading, though, the array is reserved when
 *     the library's device code is first used on a device, and that first use may
 *     allocate and synchronize inside the CUDA runtime.  So make one call on each
 *     device at initialisation, before any stream capture: a call with B = 0 (all
 *     other arguments valid, pointers may be NULL) reserves the array and looks up
 *     its address without enqueueing any work.
 *   - All calls on a device share the array, which keeps the previous call's
 *     contents (the status block is cleared at the start of each call).  Calls
 *     that overlap on the GPU (other streams, other host threads) race with each
 *     other: serialize them.
 *   - A device-side wait that runs out is recorded in the array's status block:
 *     read it with sage_noalloc_get_device_status.
 *   - Arguments, layouts and errors otherwise as sage_attn_fwd; argument errors are
 *     returned before anything is enqueued. */
SAGE_API sage_status_t sage_attn_fwd_noalloc(const void *q, const void *k, const void *v, void *o, int dtype,
                                             int layout, int B, int H, int n_q, int n_kv, int d, int causal,
                                             float sm_scale, const sage_quant_mode_t *mode, void *stream);

/* sage_get_device_status for the scratch array of sage_attn_fwd_noalloc on the
 * current device: synchronizes `stream`, reads and clears the status block of the
 * array.  *code: SAGE_OK or the first device-side error (SAGE_ERR_TIMEOUT) of the
 * calls since the last read; *site: the id of the wait that ran out (0 if none). */
SAGE_API sage_status_t sage_noalloc_get_device_status(void *stream, int *code, int *site);

/* Synchronizes `stream`, copies the workspace status block to the host and clears
 * it.  *code receives SAGE_OK or the first device-side error (SAGE_ERR_TIMEOUT);
 * *site an id of the wait that ran out (0 if none).  Returns SAGE_ERR_CUDA if the
 * copy fails. */
SAGE_API sage_status_t sage_get_device_status(void *workspace, void *stream, int *code, int *site);

/* ---- workspace views (for tests and tools; all offsets in bytes) -------------
 * The workspace holds, per query head bh = b*H + h in [0, BH = B*H) and per
 * key/value head bk = b*H_kv + h_kv in [0, BHk = B*H_kv) (BHk = BH without _gqa),
 * with Tq = ceil(n_q/128), Tk = ceil(n_kv/128), nq_pad = 128 Tq, nk_pad = 128 Tk:
 *   SAGE_WS_Q8    int8  [BH][nq_pad][d]          Q codes (pad rows 0)
 *   SAGE_WS_K8    int8  [BHk][nk_pad][d]         K codes (pad rows 0)
 *   SAGE_WS_VT8   e4m3  [BHk][d][nk_pad]         V codes, transposed (pad 0); in the
 *                                                FP16 P / V mode fp16 V, same shape
 *   SAGE_WS_DQ    fp32  [BH][nq_pad]             delta_Q of each row's group
 *   SAGE_WS_DK    fp32  [BHk][nk_pad/16]         delta_K of each 16-key run
 *   SAGE_WS_DV    fp32  [BHk][d]                 delta_V per channel
 *   SAGE_WS_QBAR  fp32  [BH][Tq][d]              Q block means
 *   SAGE_WS_KBAR  fp32  [BHk][d]                 K token mean
 *   SAGE_WS_DS    fp32  [BH][Tq][nk_pad]         dS = qbar_t . K[j] (causally
 *                                                invisible entries left unwritten)
 *   SAGE_WS_QS_KBAR fp32 [BH][nq_pad]            (q_i - qbar_t) . kbar per row: the
 *                                                shift K smoothing gives the row's logits
 *   SAGE_WS_SFQ, SAGE_WS_SFK                     E4M3 scale atoms of the SAGE_QK_FP4 mode
 *                                                (zero bytes in the other modes)
 *   SAGE_WS_LSE   fp32  [BH][nq_pad]             per row, written by the attention
 *                                                step: log-sum-exp (natural log) of the
 *                                                row's logits sm_scale q_i . k_j over its
 *                                                visible keys, as the method computes
 *                                                them (quantized scores, dS), with the K
 *                                                smoothing shift added back; -inf for a
 *                                                row that sees no key; rows >= n_q are
 *                                                not written.  It merges partial outputs
 *                                                over key ranges.
 * Along the key axis of VT8 and DS, each 128-key tile is stored in the order
 * (even keys, odd keys): key j of the tile starting at j0 is at position
 * j0 + (j & 1) * 64 + (j >> 1).  The attention kernel's threads hold the even and
 * the odd keys of a row, and PV does not depend on the order of keys.
 */
enum {
    SAGE_WS_Q8 = 0, SAGE_WS_K8 = 1, SAGE_WS_VT8 = 2, SAGE_WS_DQ = 3, SAGE_WS_DK = 4,
    SAGE_WS_DV = 5, SAGE_WS_QBAR = 6, SAGE_WS_KBAR = 7, SAGE_WS_DS = 8, SAGE_WS_QS_KBAR = 9,
    SAGE_WS_LSE = 10, SAGE_WS_SFQ = 11, SAGE_WS_SFK = 12, SAGE_WS_NUM_VIEWS = 13
};
/* Byte offset of view `which` inside the workspace, or -1 for bad arguments. */
SAGE_API int64_t sage_workspace_offset(int B, int H, int n_q, int n_kv, int d, int which);
SAGE_API int64_t sage_workspace_offset_gqa(int B, int H, int H_kv, int n_q, int n_kv, int d, int which);
SAGE_API int64_t sage_workspace_offset_mode(int B, int H, int H_kv, int n_q, int n_kv, int d,
                                            const sage_quant_mode_t *mode, int which);

/* ---- diagnostics (no counterpart on the pages' API) ---------------------------
 * INT32 scores of one (bh, Q tile, KV tile) straight from tensor memory, computed
 * by the same descriptors and tcgen05.mma kind::i8 issue as the attention kernel,
 * from a workspace filled by sage_quant_qk.  s_out: device int32 [128][128],
 * row = query row within the tile, column = key within the tile. */
SAGE_API sage_status_t sage_debug_qk_tile(const void *workspace, int B, int H, int n_q, int n_kv,
                                          int d, int bh, int q_tile, int kv_tile,
                                          int32_t *s_out, void *stream);

/* O = sum over n_tiles of P_t . V_t on the FP8 path of the attention kernel (the
 * same shared-memory layout, descriptors and tcgen05.mma kind::f8f6f4 issue, one
 * FP32 tensor-memory accumulator).  p: device E4M3 [n_tiles][128][128] (row,
 * key); vt: device E4M3 [n_tiles][d][128] (channel, key); o: device fp32
 * [128][d].  Used to check the accumulation precision of the FP8 tensor core. */
SAGE_API sage_status_t sage_debug_pv_accumulate(const uint8_t *p, const uint8_t *vt, int n_tiles,
                                                int d, float *o, void *stream);

/* The same P . V sum with an FP16 accumulator (tcgen05.mma kind::f8f6f4, D format
 * f16): the instruction SageAttention2++ moves PV to ("SageAttention2++" verdict,
 * key_machinery), whose range narrowing Pr * Vr <= 2047/2 keeps the FP16 sums finite.
 * o_raw: device uint32 [128][d], the raw 32-bit tensor-memory word of each
 * accumulator element as read by tcgen05.ld (the FP16 value's position in the word
 * is what the test establishes). */
SAGE_API sage_status_t sage_debug_pv_accumulate_f16acc(const uint8_t *p, const uint8_t *vt, int n_tiles,
                                                       int d, uint32_t *o_raw, void *stream);

/* Tensor-core throughput probe: n_ctas CTAs (one per SM) each issue n_iter
 * tcgen05.mma of M = 128, N = 256 and one 32-byte K step (K = 32 for 8-bit
 * operands, 16 for 16-bit) from zeroed shared-memory tiles into one tensor-memory
 * accumulator and wait for them.  kind: 0 E4M3 -> FP32, 1 E4M3 -> FP16, 2 S8 -> S32,
 * 3 BF16 -> FP32.  The caller times the launch on `stream`: the rate is
 * n_ctas * n_iter * 2 * 128 * 256 * K / t.  status_block: device buffer of at least
 * 256 zeroed bytes, read with sage_get_device_status (a wait that runs out records
 * SAGE_ERR_TIMEOUT).  n_iter <= 2^20, n_ctas <= 4096. */
SAGE_API sage_status_t sage_debug_mma_rate(int kind, int n_iter, int n_ctas, void *status_block, void *stream);

/* FP4 quantization of smoothed rows, the building block of the 4-bit Q / K path
 * (block-scaled E2M1 operands of tcgen05.mma kind::mxf4nvf4): per 128-row tile an fp32
 * scale g = amax / 2688 (1 if amax = 0), per row and 16 channels an E4M3 scale
 * sf = E4M3(amax / g / 6) (1.0 if amax = 0; 2^-9 if it rounds to 0), per element the
 * E2M1 code of x / (g * sf) (round to nearest even, saturating at +-6), every
 * quotient rounded to fp32.
 *   xs    : device fp32 [n_rows][d] (16-byte aligned), rows past n_rows read as 0
 *   codes : device uint8 [n_pad][d/2], two codes per byte, channel 2i in the low nibble
 *   sf    : device uint8 [n_pad][d/16], E4M3 codes
 *   g     : device fp32 [n_pad/128]
 * with n_pad = ceil(n_rows / 128) * 128. */
SAGE_API sage_status_t sage_debug_quant_fp4(const float *xs, int n_rows, int d, uint8_t *codes, uint8_t *sf,
                                            float *g, void *stream);

/* Check of the quotient routine of the quantizers (Markstein's correction of x * RN(1/delta),
 * "Computation of elementary functions on the IBM RISC System/6000 processor", 1990),
 * which stands for the IEEE fp32 division x / delta that the INT8 and E4M3 codes are
 * defined on: for every finite 16-bit pattern x of dtype (SAGE_DTYPE_BF16 or
 * SAGE_DTYPE_F16) and every deltas[j] >= 2^-60 (below that the quantizers divide)
 * with |x| <= 448 deltas[j], the routine's results for x and for -x are compared with
 * the division: bit for bit where the quotient is at least 2^-20; for every x as the
 * E4M3 codes the V
 * quantizer forms; and, where |x / deltas[j]| <= 127, as the INT8 codes the Q and K
 * quantizers form.
 *   deltas : device fp32 [n_delta], 1 <= n_delta <= 65535
 *   count  : device uint64, incremented by the number of mismatches (zero it first)
 *   first  : device uint32 [3], zeroed; on a mismatch {pattern, delta index, 1}
 * Asynchronous on `stream`; SAGE_ERR_INVALID_ARG for null pointers or a bad count or dtype. */
SAGE_API sage_status_t sage_debug_quotient_check(const float *deltas, int n_delta, int dtype, unsigned long long *count,
                                                 unsigned int *first, void *stream);

/* One 128 x 128 QK^T tile of the 4-bit mode on the block-scaled tensor core
 * (tcgen05.mma kind::mxf4nvf4, one E4M3 scale per 16 channels, scale factors copied
 * into tensor memory by tcgen05.cp):
 *   s_out[i][j] = sum over 16-channel blocks b of sfq[i][b] * sfk[j][b] *
 *                 (sum over the block's channels c of e2m1(q4[i][c]) * e2m1(k4[j][c]))
 * accumulated in FP32.  q4, k4: device uint8 [128][d/2] E2M1 codes, channel 2c in the
 * low nibble of byte c (16-byte aligned); sfq, sfk: device uint8 [128][d/16] E4M3 scale
 * codes; s_out: device fp32 [128][128] (row = query, column = key).  status_block:
 * device buffer of at least 256 zeroed bytes (read with sage_get_device_status).  The
 * per-tile fp32 scales g of the 4-bit mode multiply the result outside the tensor core. */
SAGE_API sage_status_t sage_debug_qk_tile_fp4(const uint8_t *q4, const uint8_t *k4, const uint8_t *sfq,
                                              const uint8_t *sfk, int d, float *s_out, void *status_block,
                                              void *stream);

/* Runs the attention kernel with one deliberately missing producer signal so that
 * the consumer's bounded wait must run out; the kernel records SAGE_ERR_TIMEOUT in
 * the status block and exits without hanging.  Arguments as sage_attn_fwd_prequant;
 * workspace NULL runs it on the scratch array of sage_attn_fwd_noalloc (as the last
 * call on the current device left it), whose status block
 * sage_noalloc_get_device_status reads. */
SAGE_API sage_status_t sage_debug_attn_fault_inject(void *o, int dtype, int layout, int B, int H,
                                                    int n_q, int n_kv, int d, int causal,
                                                    const void *workspace, size_t workspace_bytes,
                                                    void *stream);

/* The same for the attention kernel that quantizes Q itself (sage_attn_fwd_qfused_gqa
 * with v = NULL): q, k are the caller's 16-bit tensors and the workspace holds their K / V
 * pre-pass.  Every role of that kernel (its Q quantization, its dS warp) leaves through
 * its bounded waits.  Arguments otherwise as sage_debug_attn_fault_inject (no NULL
 * workspace). */
SAGE_API sage_status_t sage_debug_attn_fault_inject_qfused(const void *q, const void *k, void *o, int dtype,
                                                          int layout, int B, int H, int n_q, int n_kv, int d,
                                                          int causal, const void *workspace, size_t workspace_bytes,
                                                          void *stream);

/* Library build identification string (static storage). */
SAGE_API const char *sage_version(void);

#ifdef __cplusplus
}
#endif
#endif /* SAGE_B200_H */
