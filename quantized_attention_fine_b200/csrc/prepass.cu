// prepass.cu -- smoothing and quantization pre-pass of the SageAttention2-style
// forward ("SageAttention2", arXiv 2411.10958, abstract: smoothing of Q and K,
// fine-grained Q/K quantization, FP8 V; per-channel V scale from the
// pith.science verdict on arXiv 2505.21136, key_machinery).
//
// Four kernels, all bandwidth-bound except the dS product:
//   kv_stats     per (head, 512-token chunk): fp64 partial sums of K per channel
//                and per-channel max |V|.
//   kv_finalize  per head: kbar = fp32(sum / n_kv); delta_V = max|V| / Vr.
//   quant_q      per (head, 128-row block): qbar (fp64 mean of the valid rows,
//                rounded to fp32), Q_s = Q - qbar in fp32, group amax, INT8 codes.
//   quant_kv     per (head, 128-key tile): K_s = K - kbar, INT8 codes per group,
//                delta_K per 16-key run; V / delta_V -> E4M3, written transposed
//                ([channel][key]); dS[t][j] = qbar_t . K[j] for the Q blocks t
//                that can see the tile.
// Every code decision (INT8 rounding, E4M3 rounding) is an IEEE fp32 quotient
// (__fdiv_rn) rounded half to even, so that it is reproducible on the host.
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

__device__ __forceinline__ int8_t int8_code(float xs, float delta) {
    float r = rintf(__fdiv_rn(xs, delta));
    r = fminf(fmaxf(r, -127.f), 127.f);
    return (int8_t)(int)r;
}

__device__ __forceinline__ uint8_t e4m3_code(float x) {
    return (uint8_t)(pack_e4m3x4(x, 0.f, 0.f, 0.f) & 0xFFu);
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
__global__ void __launch_bounds__(256) quant_q_kernel(const PrepassArgs a) {
    constexpr int VEC = D / 32, RPW = 16;
    __shared__ double s_sum[8][D];
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
        for (int w = 0; w < 8; ++w) s = __dadd_rn(s, s_sum[w][c]);
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
        int8_t c[VEC];
#pragma unroll
        for (int v = 0; v < VEC; ++v) c[v] = int8_code(x[i][v], dl);
        store_codes<VEC>(q8 + (size_t)r * D, c);
    }
}

// ---------------------------------------------------------------------------
template <int D>
struct QuantKvSmem {
    float kt[D][kTile + 1];        // raw K of the tile, transposed (for dS)
    float qbt[D][36];              // a chunk of 32 Q block means, transposed ([channel][block])
    uint8_t vt[D][kTile + 16];     // E4M3 V codes of the tile, transposed
    float ramax[kTile];
    float delta[kTile];
};

template <int D>
__global__ void __launch_bounds__(256, 1) quant_kv_kernel(const PrepassArgs a, int ds_t_skip, int causal_off) {
    constexpr int VEC = D / 32, RPW = 16;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    QuantKvSmem<D> &sm = *reinterpret_cast<QuantKvSmem<D> *>(smem_raw);
    const Shape &S = a.shape;
    const int jt = blockIdx.x, bh = blockIdx.y;
    const int b = bh / S.H, h = bh % S.H;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int j0 = jt * kTile;
    const int nvalid = min(kTile, S.n_kv - j0);
    const bool need_ds = a.k != nullptr && a.smooth_q;

    if (a.k) {
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
            float am = 0.f;
#pragma unroll
            for (int v = 0; v < VEC; ++v) {
                if (need_ds) sm.kt[lane * VEC + v][r] = x[i][v];
                const float xs = (r < nvalid) ? __fsub_rn(x[i][v], kb[v]) : 0.f;
                x[i][v] = xs;
                am = fmaxf(am, fabsf(xs));
            }
            am = warp_max(am);
            if (lane == 0) sm.ramax[r] = am;
        }
        __syncthreads();
        if (threadIdx.x < kTile) {
            const int r = threadIdx.x;
            const int g0 = (r / a.g_k) * a.g_k;
            float am = 0.f;
            for (int rr = g0; rr < g0 + a.g_k; ++rr) am = fmaxf(am, sm.ramax[rr]);
            const float dl = (am == 0.f) ? 1.f : __fdiv_rn(am, 127.f);
            sm.delta[r] = dl;
            if ((r % kKeyRun) == 0)
                reinterpret_cast<float *>(a.ws + a.L.dk)[(size_t)bh * (S.nk_pad / kKeyRun) + (j0 + r) / kKeyRun] = dl;
        }
        __syncthreads();
        int8_t *k8 = reinterpret_cast<int8_t *>(a.ws + a.L.k8) + ((size_t)bh * S.nk_pad + j0) * D + lane * VEC;
#pragma unroll
        for (int i = 0; i < RPW; ++i) {
            const int r = warp * RPW + i;
            const float dl = sm.delta[r];
            int8_t c[VEC];
#pragma unroll
            for (int v = 0; v < VEC; ++v) c[v] = int8_code(x[i][v], dl);
            store_codes<VEC>(k8 + (size_t)r * D, c);
        }
    }

    if (a.v) {
        const uint16_t *vp = static_cast<const uint16_t *>(a.v) + b * a.skv.b + h * a.skv.h + lane * VEC;
        float dv[VEC];
#pragma unroll
        for (int v = 0; v < VEC; ++v) dv[v] = reinterpret_cast<const float *>(a.ws + a.L.dv)[(size_t)bh * D + lane * VEC + v];
#pragma unroll 4
        for (int i = 0; i < RPW; ++i) {
            const int r = warp * RPW + i;
            float x[VEC];
            if (r < nvalid) {
                load_row_slice<VEC>(vp + (int64_t)(j0 + r) * a.skv.n, a.bf16, x);
            } else {
#pragma unroll
                for (int v = 0; v < VEC; ++v) x[v] = 0.f;
            }
#pragma unroll
            for (int v = 0; v < VEC; ++v) sm.vt[lane * VEC + v][r] = e4m3_code(__fdiv_rn(x[v], dv[v]));
        }
        __syncthreads();
        uint8_t *vt8 = a.ws + a.L.vt8;
        for (int idx = threadIdx.x; idx < D * (kTile / 16); idx += blockDim.x) {
            const int c = idx / (kTile / 16), ch = idx % (kTile / 16);
            const uint4 val = *reinterpret_cast<const uint4 *>(&sm.vt[c][ch * 16]);
            *reinterpret_cast<uint4 *>(vt8 + ((size_t)bh * D + c) * S.nk_pad + j0 + ch * 16) = val;
        }
    }

    if (need_ds) {
        // dS[t][j] = qbar_t . K[j] for this tile's keys: thread (j, half) keeps K[j] in
        // registers and accumulates 8 Q blocks at a time (independent FMA chains).
        __syncthreads();
        const int j = threadIdx.x & (kTile - 1), half = threadIdx.x >> 7;
        float kr[D];
#pragma unroll
        for (int c = 0; c < D; ++c) kr[c] = sm.kt[c][j];
        int t_lo = 0;
        if (ds_t_skip) {
            const int num = j0 - causal_off - (kTile - 1);
            t_lo = num <= 0 ? 0 : (num + kTile - 1) / kTile;
            if (t_lo > S.Tq - 1) t_lo = S.Tq - 1;
        }
        const float *qbar = reinterpret_cast<const float *>(a.ws + a.L.qbar) + (size_t)bh * S.Tq * D;
        float *ds = reinterpret_cast<float *>(a.ws + a.L.ds) + (size_t)bh * S.Tq * S.nk_pad + j0 + j;
        for (int tc = t_lo; tc < S.Tq; tc += 32) {
            const int nt = min(32, S.Tq - tc);
            for (int idx = threadIdx.x; idx < 32 * D; idx += blockDim.x) {
                const int tt = idx / D, c = idx % D;
                sm.qbt[c][tt] = (tt < nt) ? qbar[(size_t)(tc + tt) * D + c] : 0.f;
            }
            __syncthreads();
#pragma unroll 1
            for (int tt0 = half * 16; tt0 < half * 16 + 16 && tt0 < nt; tt0 += 8) {
                float acc[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll
                for (int c = 0; c < D; ++c) {
                    const float4 qa = *reinterpret_cast<const float4 *>(&sm.qbt[c][tt0]);
                    const float4 qb = *reinterpret_cast<const float4 *>(&sm.qbt[c][tt0 + 4]);
                    acc[0] = fmaf(qa.x, kr[c], acc[0]);
                    acc[1] = fmaf(qa.y, kr[c], acc[1]);
                    acc[2] = fmaf(qa.z, kr[c], acc[2]);
                    acc[3] = fmaf(qa.w, kr[c], acc[3]);
                    acc[4] = fmaf(qb.x, kr[c], acc[4]);
                    acc[5] = fmaf(qb.y, kr[c], acc[5]);
                    acc[6] = fmaf(qb.z, kr[c], acc[6]);
                    acc[7] = fmaf(qb.w, kr[c], acc[7]);
                }
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    if (tt0 + i < nt) ds[(size_t)(tc + tt0 + i) * S.nk_pad] = acc[i];
            }
            __syncthreads();
        }
    }
}

// ---------------------------------------------------------------------------
template <int D>
static cudaError_t launch_prepass_d(const PrepassArgs &a, int ds_t_skip, int causal_off, cudaStream_t stream) {
    const Shape &S = a.shape;
    if (a.k || a.v) {
        kv_stats_kernel<D><<<dim3(S.n_chunks, S.BH), 256, 0, stream>>>(a);
        kv_finalize_kernel<D><<<S.BH, D, 0, stream>>>(a);
    }
    if (a.q) quant_q_kernel<D><<<dim3(S.Tq, S.BH), 256, 0, stream>>>(a);
    if (a.k || a.v) {
        const size_t smem = sizeof(QuantKvSmem<D>);
        cudaError_t e = cudaFuncSetAttribute(quant_kv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        quant_kv_kernel<D><<<dim3(S.Tk, S.BH), 256, smem, stream>>>(a, ds_t_skip, causal_off);
    }
    return cudaGetLastError();
}

cudaError_t launch_prepass(const PrepassArgs &a, int ds_t_skip, int causal_off, cudaStream_t stream) {
    if (a.shape.d == 128) return launch_prepass_d<128>(a, ds_t_skip, causal_off, stream);
    return launch_prepass_d<64>(a, ds_t_skip, causal_off, stream);
}

}  // namespace sage
