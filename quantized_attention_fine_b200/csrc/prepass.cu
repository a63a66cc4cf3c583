// prepass.cu -- smoothing and quantization pre-pass of the SageAttention2-style
// forward ("SageAttention2", arXiv 2411.10958, abstract: smoothing of Q and K,
// fine-grained Q/K quantization, FP8 V; per-channel V scale from the
// pith.science verdict on arXiv 2505.21136, key_machinery).
//
// Bandwidth-bound kernels (the dS product is in ds_gemm.cu):
//   kv_stats     per (head, 512-token chunk): fp64 partial sums of K per channel
//                and per-channel max |V|.
//   kv_finalize  per head: kbar = fp32(sum / n_kv); delta_V = max|V| / Vr.
//   quant_q      per (head, 128-row block): qbar (fp64 mean of the valid rows,
//                rounded to fp32), Q_s = Q - qbar in fp32, group amax, INT8 codes.
//   quant_k      per (head, 128-key tile): K_s = K - kbar, INT8 codes per group,
//                delta_K per 16-key run.
//   quant_v      per (head, 128-key tile): V / delta_V -> E4M3, written transposed
//                ([channel][key]).
// Every code decision (INT8 rounding, E4M3 rounding) is made on the IEEE fp32
// quotient x / delta, rounded to nearest even, so that it is reproducible on the
// host.  The quotient is formed as x * (1 / delta) when that product provably
// rounds to the same code, and by IEEE division otherwise (see fast_quotient_*).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "sage_device.cuh"
#include "sage_internal.h"

namespace sage {

namespace {

__device__ __forceinline__ float h16_to_f32(uint32_t bits, int bf16) {
    return bf16 ? __uint_as_float(bits << 16) : __half2float(__ushort_as_half((unsigned short)bits));
}

template <int VEC>
__device__ __forceinline__ void load_row_slice(const uint16_t *p, int bf16, float (&x)[VEC]) {
    if constexpr (VEC == 4) {
        const uint2 u = *reinterpret_cast<const uint2 *>(p);
        x[0] = h16_to_f32(u.x & 0xFFFFu, bf16);
        x[1] = h16_to_f32(u.x >> 16, bf16);
        x[2] = h16_to_f32(u.y & 0xFFFFu, bf16);
        x[3] = h16_to_f32(u.y >> 16, bf16);
    } else {
        const uint32_t u = *reinterpret_cast<const uint32_t *>(p);
        x[0] = h16_to_f32(u & 0xFFFFu, bf16);
        x[1] = h16_to_f32(u >> 16, bf16);
    }
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    return v;
}

// INT8 code: round-half-even of the IEEE fp32 quotient xs / delta, clamped to +-127.
// For |xs / delta| <= 128, t = RN(xs * RN(1 / delta)) lies within 2.3e-5 of the
// correctly rounded quotient, so when t is at least 2^-15 (3.05e-5) away from a
// half-integer both round to the same integer; only the rare near-tie takes the
// IEEE division.
__device__ __forceinline__ int8_t int8_code(float xs, float delta, float inv_delta) {
    const float t = xs * inv_delta;
    float r;
    if (fabsf(t - floorf(t) - 0.5f) >= 0x1p-15f) r = rintf(t);
    else r = rintf(__fdiv_rn(xs, delta));
    r = fminf(fmaxf(r, -127.f), 127.f);
    return (int8_t)(int)r;
}

// The IEEE fp32 quotient x / delta as far as its E4M3 rounding is concerned.
// t = RN(x * RN(1 / delta)) is within about 1.5 fp32 ulp of the correctly rounded
// quotient; E4M3 rounds at bit 19 of the fp32 mantissa (normal range), so unless the
// 20 low bits of t are within 4 of the tie pattern 0x80000 both round alike.  The
// subnormal E4M3 range (|t| < 2^-6) and near-ties use the IEEE division.
__device__ __forceinline__ float e4m3_quotient(float x, float delta, float inv_delta) {
    const float t = x * inv_delta;
    const int dist = (int)(__float_as_uint(t) & 0xFFFFFu) - 0x80000;
    if (fabsf(t) < 0x1p-6f || (dist >= -4 && dist <= 4)) return __fdiv_rn(x, delta);
    return t;
}

template <int VEC>
__device__ __forceinline__ void store_codes(int8_t *dst, const int8_t (&c)[VEC]) {
    if constexpr (VEC == 4) {
        uint32_t w = (uint32_t)(uint8_t)c[0] | ((uint32_t)(uint8_t)c[1] << 8) | ((uint32_t)(uint8_t)c[2] << 16) |
                     ((uint32_t)(uint8_t)c[3] << 24);
        *reinterpret_cast<uint32_t *>(dst) = w;
    } else {
        uint16_t w = (uint16_t)((uint32_t)(uint8_t)c[0] | ((uint32_t)(uint8_t)c[1] << 8));
        *reinterpret_cast<uint16_t *>(dst) = w;
    }
}

}  // namespace

// Quantization kernels: 16 warps per 128-row (or 128-key) tile, 8 rows per warp.
constexpr int kQuantThreads = 512;
constexpr int kQuantWarps = kQuantThreads / 32;
constexpr int kRowsPerWarp = kTile / kQuantWarps;

// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) kv_stats_kernel(const PrepassArgs a) {
    constexpr int VEC = D / 32;
    __shared__ double s_sum[8][D];
    __shared__ float s_max[8][D];
    const int chunk = blockIdx.x, bh = blockIdx.y;
    const int b = bh / a.shape.H, h = bh % a.shape.H;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int j0 = chunk * kStatChunk;
    const int j1 = min(j0 + kStatChunk, a.shape.n_kv);
    double ks[VEC];
    float vm[VEC];
#pragma unroll
    for (int v = 0; v < VEC; ++v) { ks[v] = 0.0; vm[v] = 0.f; }
    const uint16_t *kp = a.k ? static_cast<const uint16_t *>(a.k) + b * a.skv.b + h * a.skv.h + lane * VEC : nullptr;
    const uint16_t *vp = a.v ? static_cast<const uint16_t *>(a.v) + b * a.skv.b + h * a.skv.h + lane * VEC : nullptr;
    for (int j = j0 + warp; j < j1; j += 8) {
        float x[VEC];
        if (kp) {
            load_row_slice<VEC>(kp + (int64_t)j * a.skv.n, a.bf16, x);
#pragma unroll
            for (int v = 0; v < VEC; ++v) ks[v] = __dadd_rn(ks[v], (double)x[v]);
        }
        if (vp) {
            load_row_slice<VEC>(vp + (int64_t)j * a.skv.n, a.bf16, x);
#pragma unroll
            for (int v = 0; v < VEC; ++v) vm[v] = fmaxf(vm[v], fabsf(x[v]));
        }
    }
#pragma unroll
    for (int v = 0; v < VEC; ++v) {
        s_sum[warp][lane * VEC + v] = ks[v];
        s_max[warp][lane * VEC + v] = vm[v];
    }
    __syncthreads();
    if (threadIdx.x < D) {
        const int c = threadIdx.x;
        double s = 0.0;
        float m = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) { s = __dadd_rn(s, s_sum[w][c]); m = fmaxf(m, s_max[w][c]); }
        const size_t o = ((size_t)bh * a.shape.n_chunks + chunk) * D + c;
        if (a.k) reinterpret_cast<double *>(a.ws + a.L.ksum_part)[o] = s;
        if (a.v) reinterpret_cast<float *>(a.ws + a.L.vmax_part)[o] = m;
    }
}

template <int D>
__global__ void kv_finalize_kernel(const PrepassArgs a) {
    const int bh = blockIdx.x, c = threadIdx.x;
    const int nc = a.shape.n_chunks;
    if (a.k) {
        const double *part = reinterpret_cast<const double *>(a.ws + a.L.ksum_part) + (size_t)bh * nc * D + c;
        double s = 0.0;
        for (int ch = 0; ch < nc; ++ch) s = __dadd_rn(s, part[(size_t)ch * D]);
        const float kb = (a.smooth_k && a.shape.n_kv > 0) ? (float)__ddiv_rn(s, (double)a.shape.n_kv) : 0.f;
        reinterpret_cast<float *>(a.ws + a.L.kbar)[(size_t)bh * D + c] = kb;
    }
    if (a.v) {
        const float *part = reinterpret_cast<const float *>(a.ws + a.L.vmax_part) + (size_t)bh * nc * D + c;
        float m = 0.f;
        for (int ch = 0; ch < nc; ++ch) m = fmaxf(m, part[(size_t)ch * D]);
        reinterpret_cast<float *>(a.ws + a.L.dv)[(size_t)bh * D + c] = (m == 0.f) ? 1.f : __fdiv_rn(m, a.v_range);
    }
}

// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kQuantThreads) quant_q_kernel(const PrepassArgs a) {
    constexpr int VEC = D / 32, RPW = kRowsPerWarp;
    __shared__ double s_sum[kQuantWarps][D];
    __shared__ float s_qbar[D];
    __shared__ float s_ramax[kTile];
    __shared__ float s_delta[kTile];
    const Shape &S = a.shape;
    const int t = blockIdx.x, bh = blockIdx.y;
    const int b = bh / S.H, h = bh % S.H;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r0 = t * kTile;
    const int nvalid = min(kTile, S.n_q - r0);
    const uint16_t *qp = static_cast<const uint16_t *>(a.q) + b * a.sq.b + h * a.sq.h + lane * VEC;

    float x[RPW][VEC];
    double ps[VEC];
#pragma unroll
    for (int v = 0; v < VEC; ++v) ps[v] = 0.0;
#pragma unroll
    for (int i = 0; i < RPW; ++i) {
        const int r = warp * RPW + i;
        if (r < nvalid) {
            load_row_slice<VEC>(qp + (int64_t)(r0 + r) * a.sq.n, a.bf16, x[i]);
#pragma unroll
            for (int v = 0; v < VEC; ++v) ps[v] = __dadd_rn(ps[v], (double)x[i][v]);
        } else {
#pragma unroll
            for (int v = 0; v < VEC; ++v) x[i][v] = 0.f;
        }
    }
#pragma unroll
    for (int v = 0; v < VEC; ++v) s_sum[warp][lane * VEC + v] = ps[v];
    __syncthreads();
    if (threadIdx.x < D) {
        const int c = threadIdx.x;
        double s = 0.0;
#pragma unroll
        for (int w = 0; w < kQuantWarps; ++w) s = __dadd_rn(s, s_sum[w][c]);
        const float qb = a.smooth_q ? (float)__ddiv_rn(s, (double)nvalid) : 0.f;
        s_qbar[c] = qb;
        reinterpret_cast<float *>(a.ws + a.L.qbar)[((size_t)bh * S.Tq + t) * D + c] = qb;
    }
    __syncthreads();
    float qb[VEC];
#pragma unroll
    for (int v = 0; v < VEC; ++v) qb[v] = s_qbar[lane * VEC + v];
#pragma unroll
    for (int i = 0; i < RPW; ++i) {
        const int r = warp * RPW + i;
        float am = 0.f;
#pragma unroll
        for (int v = 0; v < VEC; ++v) {
            const float xs = (r < nvalid) ? __fsub_rn(x[i][v], qb[v]) : 0.f;
            x[i][v] = xs;
            am = fmaxf(am, fabsf(xs));
        }
        am = warp_max(am);
        if (lane == 0) s_ramax[r] = am;
    }
    __syncthreads();
    if (threadIdx.x < kTile) {
        const int r = threadIdx.x;
        const int g0 = (r / a.g_q) * a.g_q;
        float am = 0.f;
        for (int rr = g0; rr < g0 + a.g_q; ++rr) am = fmaxf(am, s_ramax[rr]);
        const float dl = (am == 0.f) ? 1.f : __fdiv_rn(am, 127.f);
        s_delta[r] = dl;
        reinterpret_cast<float *>(a.ws + a.L.dq)[(size_t)bh * S.nq_pad + r0 + r] = dl;
    }
    __syncthreads();
    int8_t *q8 = reinterpret_cast<int8_t *>(a.ws + a.L.q8) + ((size_t)bh * S.nq_pad + r0) * D + lane * VEC;
#pragma unroll
    for (int i = 0; i < RPW; ++i) {
        const int r = warp * RPW + i;
        const float dl = s_delta[r];
        const float inv = 1.0f / dl;
        int8_t c[VEC];
#pragma unroll
        for (int v = 0; v < VEC; ++v) c[v] = int8_code(x[i][v], dl, inv);
        store_codes<VEC>(q8 + (size_t)r * D, c);
    }
}

// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kQuantThreads) quant_k_kernel(const PrepassArgs a) {
    constexpr int VEC = D / 32, RPW = kRowsPerWarp;
    __shared__ float s_ramax[kTile];
    __shared__ float s_delta[kTile];
    const Shape &S = a.shape;
    const int jt = blockIdx.x, bh = blockIdx.y;
    const int b = bh / S.H, h = bh % S.H;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int j0 = jt * kTile;
    const int nvalid = min(kTile, S.n_kv - j0);
    const uint16_t *kp = static_cast<const uint16_t *>(a.k) + b * a.skv.b + h * a.skv.h + lane * VEC;
    float kb[VEC];
#pragma unroll
    for (int v = 0; v < VEC; ++v) kb[v] = reinterpret_cast<const float *>(a.ws + a.L.kbar)[(size_t)bh * D + lane * VEC + v];
    float x[RPW][VEC];
#pragma unroll
    for (int i = 0; i < RPW; ++i) {
        const int r = warp * RPW + i;
        if (r < nvalid) {
            load_row_slice<VEC>(kp + (int64_t)(j0 + r) * a.skv.n, a.bf16, x[i]);
        } else {
#pragma unroll
            for (int v = 0; v < VEC; ++v) x[i][v] = 0.f;
        }
    }
#pragma unroll
    for (int i = 0; i < RPW; ++i) {
        const int r = warp * RPW + i;
        float am = 0.f;
#pragma unroll
        for (int v = 0; v < VEC; ++v) {
            const float xs = (r < nvalid) ? __fsub_rn(x[i][v], kb[v]) : 0.f;
            x[i][v] = xs;
            am = fmaxf(am, fabsf(xs));
        }
        am = warp_max(am);
        if (lane == 0) s_ramax[r] = am;
    }
    __syncthreads();
    if (threadIdx.x < kTile) {
        const int r = threadIdx.x;
        const int g0 = (r / a.g_k) * a.g_k;
        float am = 0.f;
        for (int rr = g0; rr < g0 + a.g_k; ++rr) am = fmaxf(am, s_ramax[rr]);
        const float dl = (am == 0.f) ? 1.f : __fdiv_rn(am, 127.f);
        s_delta[r] = dl;
        if ((r % kKeyRun) == 0)
            reinterpret_cast<float *>(a.ws + a.L.dk)[(size_t)bh * (S.nk_pad / kKeyRun) + (j0 + r) / kKeyRun] = dl;
    }
    __syncthreads();
    int8_t *k8 = reinterpret_cast<int8_t *>(a.ws + a.L.k8) + ((size_t)bh * S.nk_pad + j0) * D + lane * VEC;
#pragma unroll
    for (int i = 0; i < RPW; ++i) {
        const int r = warp * RPW + i;
        const float dl = s_delta[r];
        const float inv = 1.0f / dl;
        int8_t c[VEC];
#pragma unroll
        for (int v = 0; v < VEC; ++v) c[v] = int8_code(x[i][v], dl, inv);
        store_codes<VEC>(k8 + (size_t)r * D, c);
    }
}

// V codes of one 128-key tile, written transposed: each lane holds 8 consecutive
// keys of VEC channels and stores them as one 8-byte piece of each channel's row of
// V^T ([channel][key]).
template <int D>
__global__ void __launch_bounds__(kQuantThreads) quant_v_kernel(const PrepassArgs a) {
    constexpr int VEC = D / 32, RPW = kRowsPerWarp;
    const Shape &S = a.shape;
    const int jt = blockIdx.x, bh = blockIdx.y;
    const int b = bh / S.H, h = bh % S.H;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int j0 = jt * kTile;
    const int nvalid = min(kTile, S.n_kv - j0);
    const uint16_t *vp = static_cast<const uint16_t *>(a.v) + b * a.skv.b + h * a.skv.h + lane * VEC;
    float dv[VEC], inv[VEC];
#pragma unroll
    for (int v = 0; v < VEC; ++v) {
        dv[v] = reinterpret_cast<const float *>(a.ws + a.L.dv)[(size_t)bh * D + lane * VEC + v];
        inv[v] = 1.0f / dv[v];
    }
    float x[RPW][VEC];
#pragma unroll
    for (int i = 0; i < RPW; ++i) {
        const int r = warp * RPW + i;
        if (r < nvalid) {
            load_row_slice<VEC>(vp + (int64_t)(j0 + r) * a.skv.n, a.bf16, x[i]);
        } else {
#pragma unroll
            for (int v = 0; v < VEC; ++v) x[i][v] = 0.f;
        }
    }
    uint8_t *vt8 = a.ws + a.L.vt8 + ((size_t)bh * D + lane * VEC) * S.nk_pad + j0 + warp * RPW;
    static_assert(RPW == 8, "each lane stores 8 keys of a channel as one 8-byte piece");
#pragma unroll
    for (int v = 0; v < VEC; ++v) {
        uint32_t w[2];
#pragma unroll
        for (int q = 0; q < 2; ++q)
            w[q] = pack_e4m3x4(e4m3_quotient(x[4 * q][v], dv[v], inv[v]), e4m3_quotient(x[4 * q + 1][v], dv[v], inv[v]),
                               e4m3_quotient(x[4 * q + 2][v], dv[v], inv[v]), e4m3_quotient(x[4 * q + 3][v], dv[v], inv[v]));
        *reinterpret_cast<uint2 *>(vt8 + (size_t)v * S.nk_pad) = make_uint2(w[0], w[1]);
    }
}

// ---------------------------------------------------------------------------
template <int D>
static cudaError_t launch_prepass_d(const PrepassArgs &a, cudaStream_t stream) {
    const Shape &S = a.shape;
    if (a.k || a.v) {
        kv_stats_kernel<D><<<dim3(S.n_chunks, S.BH), 256, 0, stream>>>(a);
        kv_finalize_kernel<D><<<S.BH, D, 0, stream>>>(a);
    }
    if (a.q) quant_q_kernel<D><<<dim3(S.Tq, S.BH), kQuantThreads, 0, stream>>>(a);
    if (a.k) quant_k_kernel<D><<<dim3(S.Tk, S.BH), kQuantThreads, 0, stream>>>(a);
    if (a.v) quant_v_kernel<D><<<dim3(S.Tk, S.BH), kQuantThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_prepass(const PrepassArgs &a, cudaStream_t stream) {
    if (a.shape.d == 128) return launch_prepass_d<128>(a, stream);
    return launch_prepass_d<64>(a, stream);
}

}  // namespace sage
