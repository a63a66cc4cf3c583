// sage_api.cu -- the C ABI of libsage_b200 (declared in include/sage.h):
// argument validation, workspace layout, TMA tensor-map encoding and kernel
// launches on the caller's stream.  No memory is allocated here.
#include <cudaTypedefs.h>
#include <math.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "../../include/sage.h"
#include "sage_internal.h"

using namespace sage;

namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;
// sage_debug_set_q_code_dump: forward calls that quantize Q in the attention kernel
// also write the Q codes to the workspace.
std::atomic<int> g_q_code_dump{0};

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    std::call_once(g_encode_once, [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    return g_encode;
}

struct Mode {
    int g_q, g_k, smooth_q, smooth_k;
    float p_range, v_range;
    int pv16;
    int fp4;   // 4-bit Q / K (SAGE_QK_FP4)
};

sage_status_t read_mode(const sage_quant_mode_t *m, Mode *out) {
    sage_quant_mode_t d = {SAGE_QK_PER_THREADGROUP, 1, 1, 448.f, 448.f, 0};
    if (m) d = *m;
    switch (d.gran) {
        case SAGE_QK_PER_BLOCK: out->g_q = 128; out->g_k = 128; break;
        case SAGE_QK_PER_WARP: out->g_q = 32; out->g_k = 128; break;
        case SAGE_QK_PER_THREADGROUP: out->g_q = 32; out->g_k = 16; break;
        case SAGE_QK_FP4: out->g_q = 128; out->g_k = 128; break;   // the tile scale spans the tile
        default: return SAGE_ERR_INVALID_ARG;
    }
    out->fp4 = (d.gran == SAGE_QK_FP4) ? 1 : 0;
    if (!(d.p_range > 0.f && d.p_range <= 448.f) || !(d.v_range > 0.f && d.v_range <= 448.f))
        return SAGE_ERR_INVALID_ARG;
    out->smooth_q = d.smooth_q ? 1 : 0;
    out->smooth_k = d.smooth_k ? 1 : 0;
    out->p_range = d.p_range;
    out->v_range = d.v_range;
    if (d.pv_fp16 != 0 && d.pv_fp16 != 1) return SAGE_ERR_INVALID_ARG;
    out->pv16 = d.pv_fp16;
    if (out->fp4 && out->pv16) return SAGE_ERR_UNSUPPORTED;   // the 4-bit mode pairs with FP8 P / V
    return SAGE_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Sizes shared by all entry points.  Returns SAGE_OK and fills *s, or an error.
// H query heads, H_kv key/value heads (H_kv divides H).
sage_status_t check_sizes(int B, int H, int H_kv, int n_q, int n_kv, int d, Shape *s) {
    if (B < 0 || H < 0 || n_q < 0 || n_kv < 0) return SAGE_ERR_INVALID_ARG;
    if (H_kv < 0 || (H > 0 && (H_kv == 0 || H % H_kv != 0)) || (H == 0 && H_kv != 0)) return SAGE_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return SAGE_ERR_UNSUPPORTED;
    // TMA coordinates are 32-bit signed: BH * padded length must stay below 2^31.
    const int64_t bh = (int64_t)B * H;
    const int64_t nq_pad = ((int64_t)n_q + kTile - 1) / kTile * kTile;
    const int64_t nk_pad = ((int64_t)n_kv + kTile - 1) / kTile * kTile;
    if (bh * nq_pad >= (1ll << 31) || bh * nk_pad >= (1ll << 31) || bh * d >= (1ll << 31)) return SAGE_ERR_UNSUPPORTED;
    if ((bh * ((nq_pad + kTile - 1) / kTile)) >= (1ll << 31)) return SAGE_ERR_UNSUPPORTED;
    *s = make_shape(B, H, H_kv, n_q, n_kv, d);
    return SAGE_OK;
}

sage_status_t check_ws(const Shape &s, const void *ws, size_t ws_bytes) {
    if (!ws) return SAGE_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(ws) & (kWsAlign - 1)) != 0) return SAGE_ERR_UNSUPPORTED;
    if (ws_bytes < ws_layout(s).total) return SAGE_ERR_WORKSPACE;
    return SAGE_OK;
}

bool encode_2d(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
               uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
    auto enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 2-D map of 16-bit elements (inner extent and box in elements, row pitch in bytes).
bool encode_2d16(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                 uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
    auto enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void *>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Tensor maps of the Q codes, K codes ([rows][d] bytes, 128-row boxes) and the
// transposed V codes ([BH*d][nk_pad] bytes, d x 128 boxes).
bool make_maps(const Shape &s, const uint8_t *ws, CUtensorMap *tq, CUtensorMap *tk, CUtensorMap *tv) {
    const WsLayout L = ws_layout(s);
    const uint64_t d = (uint64_t)s.d;
    // INT8 rows of d bytes (128- / 64-byte swizzle); FP4 rows of d / 2 bytes (64- / 32-byte swizzle)
    const uint64_t rb = s.fp4 ? d / 2 : d;
    const CUtensorMapSwizzle swz_qk = (rb == 128) ? CU_TENSOR_MAP_SWIZZLE_128B
                                      : (rb == 64) ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
    if (tq && !encode_2d(tq, ws + L.q8, rb, (uint64_t)s.BH * s.nq_pad, rb, (uint32_t)rb, kTile, swz_qk)) return false;
    if (tk && !encode_2d(tk, ws + L.k8, rb, (uint64_t)s.BH_kv * s.nk_pad, rb, (uint32_t)rb, kTile, swz_qk)) return false;
    if (tv && !s.pv16 &&
        !encode_2d(tv, ws + L.vt8, (uint64_t)s.nk_pad, (uint64_t)s.BH_kv * d, (uint64_t)s.nk_pad, kTile, (uint32_t)d,
                   CU_TENSOR_MAP_SWIZZLE_128B))
        return false;
    // FP16 V^T: 16-bit elements, boxes of 64 keys (one 128-byte swizzle span) x d channels
    if (tv && s.pv16 &&
        !encode_2d16(tv, ws + L.vt8, (uint64_t)s.nk_pad, (uint64_t)s.BH_kv * d, (uint64_t)s.nk_pad * 2, 64,
                     (uint32_t)d, CU_TENSOR_MAP_SWIZZLE_128B))
        return false;
    return true;
}

// Tensor map of a caller's 16-bit Q or K (`heads` heads of `n` rows per sequence, or
// a packed batch of s.total_* rows): [BH][n][d] (head-major) or [B][n][heads][d]
// (token-major; a packed batch is one batch), 64-element x `box_rows` boxes, 128-byte
// swizzle.  Rows past the end read as zero.
bool make_raw16_map(CUtensorMap *map, const void *x, int dtype, int layout, const Shape &s, int n, int total,
                    int heads, uint32_t box_rows) {
    auto enc = get_encode();
    if (!enc) return false;
    const CUtensorMapDataType dt =
        (dtype == SAGE_DTYPE_BF16) ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    const uint64_t d = (uint64_t)s.d;
    CUresult r;
    if (layout == SAGE_LAYOUT_HND && !s.varlen) {
        cuuint64_t dims[3] = {d, (uint64_t)n, (uint64_t)s.B * heads};
        cuuint64_t strides[2] = {d * 2, (uint64_t)n * d * 2};
        cuuint32_t box[3] = {64, box_rows, 1};
        cuuint32_t estr[3] = {1, 1, 1};
        r = enc(map, dt, 3, const_cast<void *>(x), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    } else {
        const uint64_t rows = s.varlen ? (uint64_t)total : (uint64_t)n;
        const uint64_t nb = s.varlen ? 1 : (uint64_t)s.B;
        cuuint64_t dims[4] = {d, (uint64_t)heads, rows, nb};
        cuuint64_t strides[3] = {d * 2, (uint64_t)heads * d * 2, rows * heads * d * 2};
        cuuint32_t box[4] = {64, 1, box_rows, 1};
        cuuint32_t estr[4] = {1, 1, 1, 1};
        r = enc(map, dt, 4, const_cast<void *>(x), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    }
    return r == CUDA_SUCCESS;
}

// The caller's K for the dS product of the pre-pass: 128-key boxes.
bool make_k16_map(CUtensorMap *map, const void *k, int dtype, int layout, const Shape &s) {
    return make_raw16_map(map, k, dtype, layout, s, s.n_kv, s.total_kv, s.H_kv, (uint32_t)kTile);
}

// Load map of a caller's 16-bit Q, K or V (n rows per head, `batches` batches): d x
// 128-row boxes, no swizzle; rows past n read as zero.
bool make_rows16_map(CUtensorMap *map, const void *x, int dtype, int layout, const Shape &s, int n, int heads,
                     int batches) {
    auto enc = get_encode();
    if (!enc) return false;
    const CUtensorMapDataType dt =
        (dtype == SAGE_DTYPE_BF16) ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    const uint64_t d = (uint64_t)s.d;
    if (layout == SAGE_LAYOUT_HND) {
        cuuint64_t dims[3] = {d, (uint64_t)n, (uint64_t)batches * heads};
        cuuint64_t strides[2] = {d * 2, (uint64_t)n * d * 2};
        cuuint32_t box[3] = {(cuuint32_t)d, (cuuint32_t)kTile, 1};
        cuuint32_t estr[3] = {1, 1, 1};
        return enc(map, dt, 3, const_cast<void *>(x), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    }
    cuuint64_t dims[4] = {d, (uint64_t)heads, (uint64_t)n, (uint64_t)batches};
    cuuint64_t strides[3] = {d * 2, (uint64_t)heads * d * 2, (uint64_t)n * heads * d * 2};
    cuuint32_t box[4] = {(cuuint32_t)d, 1, (cuuint32_t)kTile, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(map, dt, 4, const_cast<void *>(x), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

// Pre-pass of a dense batch (cu_q = cu_kv = null) or of a packed one (token-major
// [total][heads][d] tensors, per-sequence offsets cu_q, cu_kv on the device).
sage_status_t run_prepass(const void *q, const void *k, const void *v, int dtype, int layout, const Shape &s,
                          const Mode &m, uint8_t *ws, int ds_t_skip, int causal_off, const int *cu_q,
                          const int *cu_kv, cudaStream_t stream, bool ds_product = true) {
    PrepassArgs a;
    a.q = q;
    a.k = k;
    a.v = v;
    a.bf16 = (dtype == SAGE_DTYPE_BF16);
    a.nhd = (layout == SAGE_LAYOUT_NHD);
    a.cu_q = cu_q;
    a.cu_kv = cu_kv;
    const int nq_rows = s.varlen ? s.total_q : s.n_q, nkv_rows = s.varlen ? s.total_kv : s.n_kv;
    const int batches = s.varlen ? 1 : s.B;
    if (q && !make_rows16_map(&a.tm_q, q, dtype, layout, s, nq_rows, s.H, batches)) return SAGE_ERR_CUDA;
    if (k && !make_rows16_map(&a.tm_k, k, dtype, layout, s, nkv_rows, s.H_kv, batches)) return SAGE_ERR_CUDA;
    if (v && !make_rows16_map(&a.tm_v, v, dtype, layout, s, nkv_rows, s.H_kv, batches)) return SAGE_ERR_CUDA;
    if (v && !m.pv16 && !make_maps(s, ws, nullptr, nullptr, &a.tm_vt)) return SAGE_ERR_CUDA;
    a.sq = make_strides(layout, s.H, nq_rows, s.d);
    a.skv = make_strides(layout, s.H_kv, nkv_rows, s.d);
    a.shape = s;
    a.g_q = m.g_q;
    a.g_k = m.g_k;
    a.smooth_q = m.smooth_q;
    a.smooth_k = m.smooth_k;
    a.v_range = m.v_range;
    a.pv16 = m.pv16;
    a.fp4 = m.fp4;
    a.ws = ws;
    a.L = ws_layout(s);
    if (launch_prepass(a, stream) != cudaSuccess) return SAGE_ERR_CUDA;
    if (k && m.smooth_q && ds_product) {
        CUtensorMap tmk;
        if (!make_k16_map(&tmk, k, dtype, layout, s)) return SAGE_ERR_CUDA;
        if (launch_ds_gemm(tmk, reinterpret_cast<float *>(ws + a.L.ds), reinterpret_cast<const float *>(ws + a.L.qbar), s,
                           layout == SAGE_LAYOUT_NHD,
                           dtype == SAGE_DTYPE_BF16, ds_t_skip, causal_off, cu_q, cu_kv,
                           reinterpret_cast<int *>(ws + a.L.status), stream) != cudaSuccess)
            return SAGE_ERR_CUDA;
    }
    return SAGE_OK;
}

// q_raw, k_raw (both or neither): the caller's 16-bit Q and K; the kernel then
// quantizes Q itself and forms dS from K (the workspace needs only the K / V pre-pass).
sage_status_t run_attention(void *o, int dtype, int layout, const Shape &s, int causal, float sm_scale,
                            const Mode &m, const uint8_t *ws, int fault_inject, const int *cu_q, const int *cu_kv,
                            cudaStream_t stream, const void *q_raw = nullptr, const void *k_raw = nullptr) {
    CUtensorMap tq, tk, tv, tkr;
    const bool fused = q_raw != nullptr && k_raw != nullptr;
    if (!make_maps(s, ws, fused ? nullptr : &tq, &tk, &tv)) return SAGE_ERR_CUDA;
    if (fused) {
        if (!make_raw16_map(&tq, q_raw, dtype, layout, s, s.n_q, s.total_q, s.H, (uint32_t)kTile)) return SAGE_ERR_CUDA;
        if (!make_raw16_map(&tkr, k_raw, dtype, layout, s, s.n_kv, s.total_kv, s.H_kv, 16u)) return SAGE_ERR_CUDA;
    } else {
        tkr = tq;   // not read
    }
    const WsLayout L = ws_layout(s);
    const Strides so = make_strides(layout, s.H, s.varlen ? s.total_q : s.n_q, s.d);
    AttnParams p;
    p.dq = reinterpret_cast<const float *>(ws + L.dq);
    p.dk = reinterpret_cast<const float *>(ws + L.dk);
    p.dv = reinterpret_cast<const float *>(ws + L.dv);
    p.ds = reinterpret_cast<const float *>(ws + L.ds);
    p.qs_kbar = reinterpret_cast<const float *>(ws + L.qs_kbar);
    p.lse = reinterpret_cast<float *>(const_cast<uint8_t *>(ws) + L.lse);
    p.o = o;
    p.so_b = so.b;
    p.so_h = so.h;
    p.so_n = so.n;
    p.H = s.H;
    p.H_kv = s.H_kv;
    p.group = s.H / s.H_kv;
    p.n_q = s.n_q;
    p.n_kv = s.n_kv;
    p.Tq = s.Tq;
    p.Tk = s.Tk;
    p.nq_pad = s.nq_pad;
    p.nk_pad = s.nk_pad;
    p.BH = s.BH;
    p.cu_q = cu_q;
    p.cu_kv = cu_kv;
    p.total_q = s.total_q;
    p.total_kv = s.total_kv;
    p.causal = causal ? 1 : 0;
    p.use_ds = m.smooth_q;
    p.out_bf16 = (dtype == SAGE_DTYPE_BF16);
    const float scale = (sm_scale > 0.f) ? sm_scale : 1.0f / sqrtf((float)s.d);
    p.scale_log2 = scale * 1.4426950408889634f;
    p.pv16 = m.pv16;
    p.fp4 = m.fp4;
    p.sfq = ws + L.sfq;
    p.sfk = ws + L.sfk;
    p.log2_pr = m.pv16 ? 0.f : log2f(m.p_range);  // FP16 P~ is not scaled (Pr = 1)
    p.status = reinterpret_cast<int *>(const_cast<uint8_t *>(ws) + L.status);
    p.fault_inject = fault_inject;
    p.fused_q = fused ? 1 : 0;
    p.g_q = m.g_q;
    p.nhd = (layout == SAGE_LAYOUT_NHD);
    p.kbar = reinterpret_cast<const float *>(ws + L.kbar);
    p.qbar_w = reinterpret_cast<float *>(const_cast<uint8_t *>(ws) + L.qbar);
    p.dq_w = reinterpret_cast<float *>(const_cast<uint8_t *>(ws) + L.dq);
    p.q8_dump = (fused && g_q_code_dump.load()) ? reinterpret_cast<int8_t *>(const_cast<uint8_t *>(ws) + L.q8) : nullptr;
    return launch_attention(tq, tk, tv, tkr, p, s.d, stream) == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}

sage_status_t check_common(int dtype, int layout) {
    if (dtype != SAGE_DTYPE_F16 && dtype != SAGE_DTYPE_BF16) return SAGE_ERR_INVALID_ARG;
    if (layout != SAGE_LAYOUT_HND && layout != SAGE_LAYOUT_NHD) return SAGE_ERR_INVALID_ARG;
    return SAGE_OK;
}

#define SAGE_TRY(expr)                     \
    do {                                   \
        sage_status_t _st = (expr);        \
        if (_st != SAGE_OK) return _st;    \
    } while (0)

}  // namespace

namespace sage {

sage_status_t check_fwd_args(const void *q, const void *k, const void *v, const void *o, int dtype, int layout,
                             int B, int H, int H_kv, int n_q, int n_kv, int d, const sage_quant_mode_t *mode,
                             int *plan, size_t *ws_need) {
    Shape s;
    Mode m;
    *plan = kFwdNoop;
    *ws_need = 0;
    SAGE_TRY(check_common(dtype, layout));
    SAGE_TRY(check_sizes(B, H, H_kv, n_q, n_kv, d, &s));
    SAGE_TRY(read_mode(mode, &m));
    s.pv16 = m.pv16;
    s.fp4 = m.fp4;
    if (m.fp4 && d != 64) return SAGE_ERR_UNSUPPORTED;   // FP4 attention: d = 64 (tensor-memory budget)
    if (s.BH == 0 || n_q == 0) return SAGE_OK;
    if (!q || !o || (n_kv > 0 && (!k || !v))) return SAGE_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(o) || (k && !aligned16(k)) || (v && !aligned16(v))) return SAGE_ERR_UNSUPPORTED;
    if (n_kv == 0) {
        *plan = kFwdZeroOut;
        return SAGE_OK;
    }
    *plan = kFwdRun;
    *ws_need = ws_layout(s).total;
    return SAGE_OK;
}

}  // namespace sage

extern "C" {

size_t sage_workspace_bytes_gqa(int B, int H, int H_kv, int n_q, int n_kv, int d) {
    Shape s;
    if (check_sizes(B, H, H_kv, n_q, n_kv, d, &s) != SAGE_OK) return 0;
    return ws_layout(s).total;
}

size_t sage_workspace_bytes_mode(int B, int H, int H_kv, int n_q, int n_kv, int d, const sage_quant_mode_t *mode) {
    Shape s;
    Mode m;
    if (check_sizes(B, H, H_kv, n_q, n_kv, d, &s) != SAGE_OK || read_mode(mode, &m) != SAGE_OK) return 0;
    s.pv16 = m.pv16;
    s.fp4 = m.fp4;
    return ws_layout(s).total;
}

size_t sage_workspace_bytes(int B, int H, int n_q, int n_kv, int d) {
    return sage_workspace_bytes_gqa(B, H, H, n_q, n_kv, d);
}

int64_t sage_workspace_offset_mode(int B, int H, int H_kv, int n_q, int n_kv, int d, const sage_quant_mode_t *mode,
                                   int which) {
    Shape s;
    Mode m;
    if (check_sizes(B, H, H_kv, n_q, n_kv, d, &s) != SAGE_OK || read_mode(mode, &m) != SAGE_OK) return -1;
    s.pv16 = m.pv16;
    s.fp4 = m.fp4;
    const WsLayout L = ws_layout(s);
    switch (which) {
        case SAGE_WS_Q8: return (int64_t)L.q8;
        case SAGE_WS_K8: return (int64_t)L.k8;
        case SAGE_WS_VT8: return (int64_t)L.vt8;
        case SAGE_WS_DQ: return (int64_t)L.dq;
        case SAGE_WS_DK: return (int64_t)L.dk;
        case SAGE_WS_DV: return (int64_t)L.dv;
        case SAGE_WS_QBAR: return (int64_t)L.qbar;
        case SAGE_WS_KBAR: return (int64_t)L.kbar;
        case SAGE_WS_DS: return (int64_t)L.ds;
        case SAGE_WS_QS_KBAR: return (int64_t)L.qs_kbar;
        case SAGE_WS_LSE: return (int64_t)L.lse;
        case SAGE_WS_SFQ: return (int64_t)L.sfq;
        case SAGE_WS_SFK: return (int64_t)L.sfk;
        default: return -1;
    }
}

int64_t sage_workspace_offset_gqa(int B, int H, int H_kv, int n_q, int n_kv, int d, int which) {
    return sage_workspace_offset_mode(B, H, H_kv, n_q, n_kv, d, nullptr, which);
}

int64_t sage_workspace_offset(int B, int H, int n_q, int n_kv, int d, int which) {
    return sage_workspace_offset_gqa(B, H, H, n_q, n_kv, d, which);
}

sage_status_t sage_quant_qk_gqa(const void *q, const void *k, int dtype, int layout, int B, int H, int H_kv, int n_q,
                                int n_kv, int d, const sage_quant_mode_t *mode, void *workspace,
                                size_t workspace_bytes, void *stream) {
    Shape s;
    Mode m;
    SAGE_TRY(check_common(dtype, layout));
    SAGE_TRY(check_sizes(B, H, H_kv, n_q, n_kv, d, &s));
    SAGE_TRY(read_mode(mode, &m));
    s.pv16 = m.pv16;
    s.fp4 = m.fp4;
    if (s.BH == 0 || (n_q == 0 && n_kv == 0)) return SAGE_OK;
    if ((n_q > 0 && !q) || (n_kv > 0 && !k)) return SAGE_ERR_INVALID_ARG;
    if ((q && !aligned16(q)) || (k && !aligned16(k))) return SAGE_ERR_UNSUPPORTED;
    SAGE_TRY(check_ws(s, workspace, workspace_bytes));
    return run_prepass(n_q > 0 ? q : nullptr, n_kv > 0 ? k : nullptr, nullptr, dtype, layout, s, m,
                       static_cast<uint8_t *>(workspace), 0, 0, nullptr, nullptr, static_cast<cudaStream_t>(stream));
}

sage_status_t sage_quant_qk(const void *q, const void *k, int dtype, int layout, int B, int H, int n_q, int n_kv,
                            int d, const sage_quant_mode_t *mode, void *workspace, size_t workspace_bytes,
                            void *stream) {
    return sage_quant_qk_gqa(q, k, dtype, layout, B, H, H, n_q, n_kv, d, mode, workspace, workspace_bytes, stream);
}

sage_status_t sage_quant_v_gqa(const void *v, int dtype, int layout, int B, int H, int H_kv, int n_q, int n_kv,
                               int d, const sage_quant_mode_t *mode, void *workspace, size_t workspace_bytes,
                               void *stream) {
    Shape s;
    Mode m;
    SAGE_TRY(check_common(dtype, layout));
    SAGE_TRY(check_sizes(B, H, H_kv, n_q, n_kv, d, &s));
    SAGE_TRY(read_mode(mode, &m));
    s.pv16 = m.pv16;
    s.fp4 = m.fp4;
    if (s.BH == 0 || n_kv == 0) return SAGE_OK;
    if (!v) return SAGE_ERR_INVALID_ARG;
    if (!aligned16(v)) return SAGE_ERR_UNSUPPORTED;
    SAGE_TRY(check_ws(s, workspace, workspace_bytes));
    return run_prepass(nullptr, nullptr, v, dtype, layout, s, m, static_cast<uint8_t *>(workspace), 0, 0, nullptr,
                       nullptr, static_cast<cudaStream_t>(stream));
}

sage_status_t sage_quant_v(const void *v, int dtype, int layout, int B, int H, int n_q, int n_kv, int d,
                           const sage_quant_mode_t *mode, void *workspace, size_t workspace_bytes, void *stream) {
    return sage_quant_v_gqa(v, dtype, layout, B, H, H, n_q, n_kv, d, mode, workspace, workspace_bytes, stream);
}

sage_status_t sage_attn_fwd_prequant_gqa(void *o, int dtype, int layout, int B, int H, int H_kv, int n_q,
                                         int n_kv, int d, int causal, float sm_scale,
                                         const sage_quant_mode_t *mode, const void *workspace,
                                         size_t workspace_bytes, void *stream) {
    Shape s;
    Mode m;
    SAGE_TRY(check_common(dtype, layout));
    SAGE_TRY(check_sizes(B, H, H_kv, n_q, n_kv, d, &s));
    SAGE_TRY(read_mode(mode, &m));
    s.pv16 = m.pv16;
    s.fp4 = m.fp4;
    if (m.fp4 && d != 64) return SAGE_ERR_UNSUPPORTED;   // FP4 attention: d = 64 (tensor-memory budget)
    if (s.BH == 0 || n_q == 0) return SAGE_OK;
    if (!o) return SAGE_ERR_INVALID_ARG;
    if (!aligned16(o)) return SAGE_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (n_kv == 0)
        return cudaMemsetAsync(o, 0, (size_t)s.BH * n_q * d * 2, st) == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
    SAGE_TRY(check_ws(s, workspace, workspace_bytes));
    return run_attention(o, dtype, layout, s, causal, sm_scale, m, static_cast<const uint8_t *>(workspace), 0, nullptr,
                         nullptr, st);
}

sage_status_t sage_attn_fwd_prequant(void *o, int dtype, int layout, int B, int H, int n_q, int n_kv, int d,
                                     int causal, float sm_scale, const sage_quant_mode_t *mode,
                                     const void *workspace, size_t workspace_bytes, void *stream) {
    return sage_attn_fwd_prequant_gqa(o, dtype, layout, B, H, H, n_q, n_kv, d, causal, sm_scale, mode, workspace,
                                      workspace_bytes, stream);
}

sage_status_t sage_attn_fwd_gqa(const void *q, const void *k, const void *v, void *o, int dtype, int layout, int B,
                                int H, int H_kv, int n_q, int n_kv, int d, int causal, float sm_scale,
                                const sage_quant_mode_t *mode, void *workspace, size_t workspace_bytes,
                                void *stream) {
    int plan = kFwdNoop;
    size_t need = 0;
    SAGE_TRY(check_fwd_args(q, k, v, o, dtype, layout, B, H, H_kv, n_q, n_kv, d, mode, &plan, &need));
    if (plan == kFwdNoop) return SAGE_OK;
    Shape s;
    Mode m;
    check_sizes(B, H, H_kv, n_q, n_kv, d, &s);   // both validated by check_fwd_args
    read_mode(mode, &m);
    s.pv16 = m.pv16;
    s.fp4 = m.fp4;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (plan == kFwdZeroOut)
        return cudaMemsetAsync(o, 0, (size_t)s.BH * n_q * d * 2, st) == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
    SAGE_TRY(check_ws(s, workspace, workspace_bytes));
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    SAGE_TRY(run_prepass(q, k, v, dtype, layout, s, m, ws, causal ? 1 : 0, n_kv - n_q, nullptr, nullptr, st));
    return run_attention(o, dtype, layout, s, causal, sm_scale, m, ws, 0, nullptr, nullptr, st);
}

sage_status_t sage_attn_fwd_qfused_gqa(const void *q, const void *k, const void *v, void *o, int dtype, int layout,
                                       int B, int H, int H_kv, int n_q, int n_kv, int d, int causal, float sm_scale,
                                       const sage_quant_mode_t *mode, void *workspace, size_t workspace_bytes,
                                       void *stream) {
    int plan = kFwdNoop;
    size_t need = 0;
    // the whole forward's checks (without v, k stands in for it: only the attention runs)
    SAGE_TRY(check_fwd_args(q, k, v ? v : k, o, dtype, layout, B, H, H_kv, n_q, n_kv, d, mode, &plan, &need));
    Shape s;
    Mode m;
    check_sizes(B, H, H_kv, n_q, n_kv, d, &s);
    read_mode(mode, &m);
    if (m.fp4) return SAGE_ERR_UNSUPPORTED;   // the 4-bit mode quantizes Q in the pre-pass
    if (plan == kFwdNoop) return SAGE_OK;
    s.pv16 = m.pv16;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (plan == kFwdZeroOut)
        return cudaMemsetAsync(o, 0, (size_t)s.BH * n_q * d * 2, st) == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
    SAGE_TRY(check_ws(s, workspace, workspace_bytes));
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    // K / V pre-pass (no Q quantization, no dS product), then attention with Q quantized
    // and dS formed in the kernel
    if (v) SAGE_TRY(run_prepass(nullptr, k, v, dtype, layout, s, m, ws, 0, 0, nullptr, nullptr, st, false));
    return run_attention(o, dtype, layout, s, causal, sm_scale, m, ws, 0, nullptr, nullptr, st, q, k);
}

sage_status_t sage_debug_set_q_code_dump(int enable) {
    if (enable != 0 && enable != 1) return SAGE_ERR_INVALID_ARG;
    g_q_code_dump.store(enable);
    return SAGE_OK;
}

sage_status_t sage_attn_fwd(const void *q, const void *k, const void *v, void *o, int dtype, int layout, int B,
                            int H, int n_q, int n_kv, int d, int causal, float sm_scale,
                            const sage_quant_mode_t *mode, void *workspace, size_t workspace_bytes, void *stream) {
    return sage_attn_fwd_gqa(q, k, v, o, dtype, layout, B, H, H, n_q, n_kv, d, causal, sm_scale, mode, workspace,
                             workspace_bytes, stream);
}

size_t sage_workspace_bytes_varlen(int B, int H, int H_kv, int max_seqlen_q, int max_seqlen_kv, int d) {
    return sage_workspace_bytes_gqa(B, H, H_kv, max_seqlen_q, max_seqlen_kv, d);
}

static sage_status_t attn_fwd_varlen_impl(const void *q, const void *k, const void *v, void *o, int dtype,
                                          const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_kv, int B, int H,
                                          int H_kv, int total_q, int total_kv, int max_seqlen_q, int max_seqlen_kv,
                                          int d, int causal, float sm_scale, const sage_quant_mode_t *mode,
                                          void *workspace, size_t workspace_bytes, void *stream, bool fuse_q) {
    Shape s;
    Mode m;
    SAGE_TRY(check_common(dtype, SAGE_LAYOUT_NHD));
    if (total_q < 0 || total_kv < 0 || total_q > (1 << 30) || total_kv > (1 << 30)) return SAGE_ERR_INVALID_ARG;
    SAGE_TRY(check_sizes(B, H, H_kv, max_seqlen_q, max_seqlen_kv, d, &s));
    SAGE_TRY(read_mode(mode, &m));
    s.pv16 = m.pv16;
    s.fp4 = m.fp4;
    if (m.fp4 && d != 64) return SAGE_ERR_UNSUPPORTED;   // FP4 attention: d = 64 (tensor-memory budget)
    s.varlen = 1;
    s.total_q = total_q;
    s.total_kv = total_kv;
    if (s.BH == 0 || total_q == 0 || max_seqlen_q == 0) return SAGE_OK;
    if (!q || !o || !cu_seqlens_q || !cu_seqlens_kv) return SAGE_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(o)) return SAGE_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (total_kv == 0 || max_seqlen_kv == 0)
        return cudaMemsetAsync(o, 0, (size_t)total_q * H * d * 2, st) == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
    if (!k || !v) return SAGE_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(v)) return SAGE_ERR_UNSUPPORTED;
    SAGE_TRY(check_ws(s, workspace, workspace_bytes));
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    if (fuse_q && !m.fp4) {   // K / V pre-pass, then attention with Q quantized in the kernel
        SAGE_TRY(run_prepass(nullptr, k, v, dtype, SAGE_LAYOUT_NHD, s, m, ws, 0, 0, cu_seqlens_q, cu_seqlens_kv, st,
                             false));
        return run_attention(o, dtype, SAGE_LAYOUT_NHD, s, causal, sm_scale, m, ws, 0, cu_seqlens_q, cu_seqlens_kv, st,
                             q, k);
    }
    SAGE_TRY(run_prepass(q, k, v, dtype, SAGE_LAYOUT_NHD, s, m, ws, causal ? 1 : 0, 0, cu_seqlens_q, cu_seqlens_kv,
                         st));
    return run_attention(o, dtype, SAGE_LAYOUT_NHD, s, causal, sm_scale, m, ws, 0, cu_seqlens_q, cu_seqlens_kv, st);
}

sage_status_t sage_attn_fwd_varlen(const void *q, const void *k, const void *v, void *o, int dtype,
                                   const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_kv, int B, int H, int H_kv,
                                   int total_q, int total_kv, int max_seqlen_q, int max_seqlen_kv, int d, int causal,
                                   float sm_scale, const sage_quant_mode_t *mode, void *workspace,
                                   size_t workspace_bytes, void *stream) {
    return attn_fwd_varlen_impl(q, k, v, o, dtype, cu_seqlens_q, cu_seqlens_kv, B, H, H_kv, total_q, total_kv,
                                max_seqlen_q, max_seqlen_kv, d, causal, sm_scale, mode, workspace, workspace_bytes,
                                stream, false);
}

sage_status_t sage_attn_fwd_varlen_qfused(const void *q, const void *k, const void *v, void *o, int dtype,
                                          const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_kv, int B, int H,
                                          int H_kv, int total_q, int total_kv, int max_seqlen_q, int max_seqlen_kv,
                                          int d, int causal, float sm_scale, const sage_quant_mode_t *mode,
                                          void *workspace, size_t workspace_bytes, void *stream) {
    sage_quant_mode_t md = {SAGE_QK_PER_THREADGROUP, 1, 1, 448.f, 448.f, 0};
    if (mode) md = *mode;
    if (md.gran == SAGE_QK_FP4) return SAGE_ERR_UNSUPPORTED;   // the 4-bit mode quantizes Q in the pre-pass
    return attn_fwd_varlen_impl(q, k, v, o, dtype, cu_seqlens_q, cu_seqlens_kv, B, H, H_kv, total_q, total_kv,
                                max_seqlen_q, max_seqlen_kv, d, causal, sm_scale, mode, workspace, workspace_bytes,
                                stream, true);
}

sage_status_t sage_get_device_status(void *workspace, void *stream, int *code, int *site) {
    if (!workspace || !code || !site) return SAGE_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int host[2] = {0, 0};
    if (cudaStreamSynchronize(st) != cudaSuccess) return SAGE_ERR_CUDA;
    if (cudaMemcpyAsync(host, workspace, sizeof(host), cudaMemcpyDeviceToHost, st) != cudaSuccess) return SAGE_ERR_CUDA;
    if (cudaMemsetAsync(workspace, 0, sizeof(host), st) != cudaSuccess) return SAGE_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return SAGE_ERR_CUDA;
    *code = host[0];
    *site = host[1];
    return SAGE_OK;
}

sage_status_t sage_debug_qk_tile(const void *workspace, int B, int H, int n_q, int n_kv, int d, int bh, int q_tile,
                                 int kv_tile, int32_t *s_out, void *stream) {
    Shape s;
    SAGE_TRY(check_sizes(B, H, H, n_q, n_kv, d, &s));
    if (!workspace || !s_out || s.BH == 0 || n_q == 0 || n_kv == 0) return SAGE_ERR_INVALID_ARG;
    if (bh < 0 || bh >= s.BH || q_tile < 0 || q_tile >= s.Tq || kv_tile < 0 || kv_tile >= s.Tk)
        return SAGE_ERR_INVALID_ARG;
    if (!aligned16(s_out)) return SAGE_ERR_UNSUPPORTED;
    const uint8_t *ws = static_cast<const uint8_t *>(workspace);
    CUtensorMap tq, tk;
    if (!make_maps(s, ws, &tq, &tk, nullptr)) return SAGE_ERR_CUDA;
    int *status = reinterpret_cast<int *>(const_cast<uint8_t *>(ws) + ws_layout(s).status);
    return launch_debug_qk_tile(tq, tk, d, bh * s.nq_pad + q_tile * kTile, bh * s.nk_pad + kv_tile * kTile, s_out,
                                status, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? SAGE_OK
               : SAGE_ERR_CUDA;
}

sage_status_t sage_debug_pv_accumulate(const uint8_t *p, const uint8_t *vt, int n_tiles, int d, float *o,
                                       void *stream) {
    if (!p || !vt || !o || n_tiles < 1) return SAGE_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return SAGE_ERR_UNSUPPORTED;
    if (!aligned16(p) || !aligned16(vt) || !aligned16(o)) return SAGE_ERR_UNSUPPORTED;
    return launch_debug_pv(p, vt, n_tiles, d, o, nullptr, static_cast<cudaStream_t>(stream), 0) == cudaSuccess
               ? SAGE_OK
               : SAGE_ERR_CUDA;
}

sage_status_t sage_debug_pv_accumulate_f16acc(const uint8_t *p, const uint8_t *vt, int n_tiles, int d,
                                              uint32_t *o_raw, void *stream) {
    if (!p || !vt || !o_raw || n_tiles < 1) return SAGE_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return SAGE_ERR_UNSUPPORTED;
    if (!aligned16(p) || !aligned16(vt) || !aligned16(o_raw)) return SAGE_ERR_UNSUPPORTED;
    return launch_debug_pv(p, vt, n_tiles, d, reinterpret_cast<float *>(o_raw), nullptr,
                           static_cast<cudaStream_t>(stream), 1) == cudaSuccess
               ? SAGE_OK
               : SAGE_ERR_CUDA;
}

sage_status_t sage_debug_mma_rate(int kind, int n_iter, int n_ctas, void *status_block, void *stream) {
    if (kind < 0 || kind > 3 || n_iter < 1 || n_iter > (1 << 20) || n_ctas < 1 || n_ctas > 4096 || !status_block)
        return SAGE_ERR_INVALID_ARG;
    return launch_debug_mma_rate(kind, n_iter, n_ctas, static_cast<int *>(status_block),
                                 static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? SAGE_OK
               : SAGE_ERR_CUDA;
}

sage_status_t sage_debug_quotient_check(const float *deltas, int n_delta, int dtype, unsigned long long *count,
                                       unsigned int *first, void *stream) {
    if (!deltas || !count || !first || n_delta < 1 || n_delta > 65535) return SAGE_ERR_INVALID_ARG;
    if (dtype != SAGE_DTYPE_BF16 && dtype != SAGE_DTYPE_F16) return SAGE_ERR_INVALID_ARG;
    return launch_debug_quotient_check(deltas, n_delta, dtype == SAGE_DTYPE_BF16 ? 1 : 0, count, first,
                                       static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? SAGE_OK
               : SAGE_ERR_CUDA;
}

sage_status_t sage_debug_quant_fp4(const float *xs, int n_rows, int d, uint8_t *codes, uint8_t *sf, float *g,
                                   void *stream) {
    if (!xs || !codes || !sf || !g || n_rows < 1 || n_rows > (1 << 24)) return SAGE_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return SAGE_ERR_UNSUPPORTED;
    if (!aligned16(xs)) return SAGE_ERR_UNSUPPORTED;
    return launch_debug_quant_fp4(xs, n_rows, d, codes, sf, g, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? SAGE_OK
               : SAGE_ERR_CUDA;
}

sage_status_t sage_debug_qk_tile_fp4(const uint8_t *q4, const uint8_t *k4, const uint8_t *sfq, const uint8_t *sfk,
                                     int d, float *s_out, void *status_block, void *stream) {
    if (!q4 || !k4 || !sfq || !sfk || !s_out || !status_block) return SAGE_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return SAGE_ERR_UNSUPPORTED;
    if (!aligned16(q4) || !aligned16(k4) || !aligned16(s_out)) return SAGE_ERR_UNSUPPORTED;
    return launch_debug_qk_fp4(q4, k4, sfq, sfk, d, s_out, static_cast<int *>(status_block),
                               static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? SAGE_OK
               : SAGE_ERR_CUDA;
}

sage_status_t sage_debug_attn_fault_inject_qfused(const void *q, const void *k, void *o, int dtype, int layout, int B,
                                                  int H, int n_q, int n_kv, int d, int causal, const void *workspace,
                                                  size_t workspace_bytes, void *stream) {
    Shape s;
    Mode m;
    SAGE_TRY(check_common(dtype, layout));
    SAGE_TRY(check_sizes(B, H, H, n_q, n_kv, d, &s));
    SAGE_TRY(read_mode(nullptr, &m));
    if (!q || !k || !o || !workspace || s.BH == 0 || n_q == 0 || n_kv == 0) return SAGE_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(o)) return SAGE_ERR_UNSUPPORTED;
    SAGE_TRY(check_ws(s, workspace, workspace_bytes));
    return run_attention(o, dtype, layout, s, causal, 0.f, m, static_cast<const uint8_t *>(workspace), 1, nullptr,
                         nullptr, static_cast<cudaStream_t>(stream), q, k);
}

sage_status_t sage_debug_attn_fault_inject(void *o, int dtype, int layout, int B, int H, int n_q, int n_kv, int d,
                                           int causal, const void *workspace, size_t workspace_bytes,
                                           void *stream) {
    Shape s;
    Mode m;
    SAGE_TRY(check_common(dtype, layout));
    SAGE_TRY(check_sizes(B, H, H, n_q, n_kv, d, &s));
    SAGE_TRY(read_mode(nullptr, &m));
    if (!o || s.BH == 0 || n_q == 0 || n_kv == 0) return SAGE_ERR_INVALID_ARG;
    if (!workspace) {  // the scratch array of sage_attn_fwd_noalloc, as its last call left it
        uint8_t *ws = nullptr;
        SAGE_TRY(noalloc_workspace(&ws, &workspace_bytes));
        workspace = ws;
    }
    SAGE_TRY(check_ws(s, workspace, workspace_bytes));
    return run_attention(o, dtype, layout, s, causal, 0.f, m, static_cast<const uint8_t *>(workspace), 1, nullptr,
                         nullptr, static_cast<cudaStream_t>(stream));
}

const char *sage_version(void) { return "libsage_b200 1.0 (sm_100a; tcgen05 INT8 QK / FP8 PV)"; }

}  // extern "C"
