// ds_gemm.cu -- the Q-smoothing bias dS[t][j] = qbar_t . K[j] on the tensor core
// ("SageAttention2", arXiv 2411.10958, abstract: smoothing Q and adding the
// difference back).
//
// Per head this is a [Tq x d] x [d x N_kv] product.  K enters exactly, in its own
// 16-bit type (bf16 or fp16), loaded by TMA straight from the caller's tensor.  The
// fp32 block means are split into two numbers of that type, qbar = hi + lo (hi the
// rounded qbar, lo the rounded remainder), so that
//     dS = K . hi^T + K . lo^T
// accumulated in fp32 tensor memory carries qbar to about 2^-17 relative for bf16
// and 2^-22 for fp16.  tcgen05.mma kind::f16, M = 128 keys, N = up to 256 Q
// blocks, K = 16 channels per instruction; D[key][block] in tensor memory, read
// back by eight warps (lane quadrant = warp % 4, alternate 32-column chunks by
// warp / 4) and written as dS[block][key] (coalesced along keys).
// Entries of Q blocks that can never see a key tile (causal) are not written.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "sage_device.cuh"
#include "sage_internal.h"

namespace sage {

constexpr int kDsThreads = 256;
constexpr int kDsTilesPerCta = 8;
constexpr int kDsMaxN = 256;
constexpr uint64_t kDsDrainNs = 50ull * 1000ull * 1000ull;

template <int D>
struct __align__(1024) DsSmem {
    static constexpr int KA = D / 64;              // 128-byte (64-element) atoms along d
    uint8_t qhi[KA][kDsMaxN * 128];
    uint8_t qlo[KA][kDsMaxN * 128];
    uint8_t k[2][KA][kTile * 128];
    uint64_t bar_k[2], bar_mma;
    uint32_t tmem_base;
    int abort_flag;
};

__device__ __forceinline__ uint32_t pack_16x2(float a, float b, bool bf16) {
    if (bf16) {
        __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
        return *reinterpret_cast<uint32_t *>(&h);
    }
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ float round16(float a, bool bf16) {
    return bf16 ? __bfloat162float(__float2bfloat16_rn(a)) : __half2float(__float2half_rn(a));
}

template <int D>
__global__ void __launch_bounds__(kDsThreads, 1)
    ds_gemm_kernel(const __grid_constant__ CUtensorMap tm_k, const float *__restrict__ qbar, float *__restrict__ ds,
                   int BH, int H, int Tq, int Tk, int n_q, int n_kv, int nk_pad, int nhd, int bf16, int causal_skip,
                   int causal_off, int *status) {
    constexpr int KA = D / 64;
    extern __shared__ uint8_t smem_raw[];
    DsSmem<D> &sm = *reinterpret_cast<DsSmem<D> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.y;
    const int jt0 = blockIdx.x * kDsTilesPerCta;
    const int n_kt = min(kDsTilesPerCta, Tk - jt0);
    const bool is_bf16 = bf16 != 0;

    if (threadIdx.x == 0) {
        mbar_init(&sm.bar_k[0], 1);
        mbar_init(&sm.bar_k[1], 1);
        mbar_init(&sm.bar_mma, 1);
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) { tmem_alloc(&sm.tmem_base, 256); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    volatile int *abort_flag = &sm.abort_flag;
    const int b = bh / H, h = bh % H;

    auto load_k = [&](int i, int buf) {
        const int j0 = (jt0 + i) * kTile;
        mbar_arrive_expect_tx(&sm.bar_k[buf], KA * kTile * 128);
        for (int a = 0; a < KA; ++a) {
            if (nhd) tma_load_4d(sm.k[buf][a], &tm_k, &sm.bar_k[buf], a * 64, h, j0, b);
            else tma_load_3d(sm.k[buf][a], &tm_k, &sm.bar_k[buf], a * 64, j0, bh);
        }
    };

    uint32_t k_phase[2] = {0, 0}, mma_phase = 0;
    bool ok = true;
    for (int tc = 0; tc < Tq && ok; tc += kDsMaxN) {
        const int nt = min(kDsMaxN, Tq - tc);
        const int N = (nt + 15) / 16 * 16;
        // --- stage qbar[tc .. tc + N) as hi / lo 16-bit K-major operands (128-byte swizzle)
        const float *qsrc = qbar + ((size_t)bh * Tq + tc) * D;
        for (int idx = threadIdx.x; idx < N * (D / 8); idx += kDsThreads) {
            const int n = idx / (D / 8), c8 = idx % (D / 8);
            float v[8];
            if (n < nt) {
                const float4 x0 = *reinterpret_cast<const float4 *>(qsrc + (size_t)n * D + c8 * 8);
                const float4 x1 = *reinterpret_cast<const float4 *>(qsrc + (size_t)n * D + c8 * 8 + 4);
                v[0] = x0.x; v[1] = x0.y; v[2] = x0.z; v[3] = x0.w; v[4] = x1.x; v[5] = x1.y; v[6] = x1.z; v[7] = x1.w;
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) v[e] = 0.f;
            }
            float hi[8], lo[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) { hi[e] = round16(v[e], is_bf16); lo[e] = v[e] - hi[e]; }
            const int a = c8 / 8, chunk = c8 % 8;
            const uint32_t off = sw128_offset((uint32_t)n, (uint32_t)chunk);
            *reinterpret_cast<uint4 *>(sm.qhi[a] + off) =
                make_uint4(pack_16x2(hi[0], hi[1], is_bf16), pack_16x2(hi[2], hi[3], is_bf16),
                           pack_16x2(hi[4], hi[5], is_bf16), pack_16x2(hi[6], hi[7], is_bf16));
            *reinterpret_cast<uint4 *>(sm.qlo[a] + off) =
                make_uint4(pack_16x2(lo[0], lo[1], is_bf16), pack_16x2(lo[2], lo[3], is_bf16),
                           pack_16x2(lo[4], lo[5], is_bf16), pack_16x2(lo[6], lo[7], is_bf16));
        }
        fence_proxy_async_smem();
        __syncthreads();
        if (threadIdx.x == 0) {
            load_k(0, 0);
            if (n_kt > 1) load_k(1, 1);
        }
        const uint32_t idesc = idesc_f16_f32(128, N, is_bf16);
        for (int i = 0; i < n_kt; ++i) {
            const int buf = i & 1;
            if (threadIdx.x == 0) {
                if (mbar_wait(&sm.bar_k[buf], k_phase[buf], abort_flag, status, 21)) {
                    tc_fence_after();
                    int step = 0;
#pragma unroll
                    for (int a = 0; a < KA; ++a) {
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk, ++step) {
                            const uint64_t ad = smem_desc(smem_u32(sm.k[buf][a]) + kk * 32, 1024u, 2u);
                            const uint64_t bh_d = smem_desc(smem_u32(sm.qhi[a]) + kk * 32, 1024u, 2u);
                            const uint64_t bl_d = smem_desc(smem_u32(sm.qlo[a]) + kk * 32, 1024u, 2u);
                            mma_f16_ss(tmem, ad, bh_d, idesc, step > 0 ? 1u : 0u);
                            mma_f16_ss(tmem, ad, bl_d, idesc, 1u);
                        }
                    }
                }
                mma_commit(&sm.bar_mma);
            }
            k_phase[buf] ^= 1;
            __syncwarp();
            mbar_wait(&sm.bar_mma, mma_phase, abort_flag, status, 22);
            mma_phase ^= 1;
            tc_fence_after();
            __syncthreads();
            if (*abort_flag) { ok = false; break; }
            // --- epilogue: D[key][block] -> dS[block][key]
            const int jt = jt0 + i;
            int t_lo = 0;
            if (causal_skip) {
                const int num = jt * kTile - causal_off - (kTile - 1);
                t_lo = num <= 0 ? 0 : (num + kTile - 1) / kTile;
                if (t_lo > Tq - 1) t_lo = Tq - 1;
            }
            const int wq = warp & 3;
            const int key = jt * kTile + wq * 32 + lane;
            float *dst = ds + (size_t)bh * Tq * nk_pad + key;
            for (int c0 = (warp >> 2) * 32; c0 < N; c0 += 64) {
                uint32_t v[32];
                tmem_ld32(tmem + ((uint32_t)(wq * 32) << 16) + c0, v);
                tmem_wait_ld_regs(v);
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int t = tc + c0 + e;
                    if (c0 + e < nt && t >= t_lo) dst[(size_t)t * nk_pad] = __uint_as_float(v[e]);
                }
            }
            tc_fence_before();
            __syncthreads();   // TMEM read and K buffer consumed
            if (threadIdx.x == 0 && i + 2 < n_kt) load_k(i + 2, buf);
        }
        if (!ok && threadIdx.x == 0) {   // let the copies in flight land before the CTA exits
            for (int i2 = 0; i2 < 2; ++i2) mbar_wait_quiet(&sm.bar_k[i2], k_phase[i2], kDsDrainNs);
        }
        __syncthreads();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) { __syncwarp(); tc_fence_after(); tmem_dealloc(tmem, 256); }
}

cudaError_t launch_ds_gemm(const CUtensorMap &tm_k, const float *qbar, float *ds, const Shape &s, int nhd, int bf16,
                           int causal_skip, int causal_off, int *status, cudaStream_t stream) {
    dim3 grid((s.Tk + kDsTilesPerCta - 1) / kDsTilesPerCta, s.BH);
    if (s.d == 128) {
        const size_t smem = sizeof(DsSmem<128>) + 1024;
        cudaError_t e = cudaFuncSetAttribute(ds_gemm_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        ds_gemm_kernel<128><<<grid, kDsThreads, smem, stream>>>(tm_k, qbar, ds, s.BH, s.H, s.Tq, s.Tk, s.n_q, s.n_kv,
                                                                 s.nk_pad, nhd, bf16, causal_skip, causal_off, status);
    } else {
        const size_t smem = sizeof(DsSmem<64>) + 1024;
        cudaError_t e = cudaFuncSetAttribute(ds_gemm_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        ds_gemm_kernel<64><<<grid, kDsThreads, smem, stream>>>(tm_k, qbar, ds, s.BH, s.H, s.Tq, s.Tk, s.n_q, s.n_kv,
                                                                s.nk_pad, nhd, bf16, causal_skip, causal_off, status);
    }
    return cudaGetLastError();
}

}  // namespace sage
