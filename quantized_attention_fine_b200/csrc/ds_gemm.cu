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
// blocks, K = 16 channels per instruction; D[key][block] in tensor memory (two
// accumulators, so the product of one key tile overlaps the write-out of the
// previous one), transposed through shared memory and written as dS[block][position]
// by TMA stores, keys of each 128-key tile in the storage order (even, then odd).
// 32-block chunks whose blocks can never see a key tile (causal) are not written.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "sage_device.cuh"
#include "sage_internal.h"

namespace sage {

constexpr int kDsThreads = 256;
constexpr int kDsTilesPerCta = 16;   // key tiles per CTA at most (fewer when that leaves SMs idle)
constexpr int kDsMaxN = 256;
constexpr int kDsChunk = 32;   // Q blocks per epilogue store box
constexpr uint64_t kDsDrainNs = 50ull * 1000ull * 1000ull;

// Roles (256 threads): warp 0 loads K tiles (TMA, two buffers); warp 1 issues the
// MMAs into one of two 256-column tensor-memory accumulators, so the product of
// key tile i + 1 overlaps the epilogue of tile i; warps 4-7 (one per lane
// quadrant) move each 32-block chunk of D[key][block] through shared memory,
// transposed to [block][key], and write it with a TMA store.  All 256 threads
// stage qbar.
template <int D>
struct __align__(1024) DsSmem {
    static constexpr int KA = D / 64;              // 128-byte (64-element) atoms along d
    uint8_t qhi[KA][kDsMaxN * 128];
    uint8_t qlo[KA][kDsMaxN * 128];
    uint8_t k[2][KA][kTile * 128];
    float stage[2][kDsChunk][kTile];
    uint64_t bar_kfull[2], bar_kempty[2], bar_afull[2], bar_aempty[2];
    uint64_t bar_stage_full[2], bar_stage_free[2];
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
    ds_gemm_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_ds,
                   const float *__restrict__ qbar, int H, int H_kv, int Tq, int Tk, int nhd, int bf16, int causal_skip,
                   int causal_off, const int *__restrict__ cu_q, const int *__restrict__ cu_kv, int n_q_max,
                   int n_kv_max, int total_q, int total_kv, int tiles_per_cta, int ctas_per_head, int *status) {
    constexpr int KA = D / 64;
    extern __shared__ uint8_t smem_raw[];
    DsSmem<D> &sm = *reinterpret_cast<DsSmem<D> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // one-dimensional grid (head-major), so any head count fits: block = bh * ctas_per_head + x
    const int bh = (int)(blockIdx.x / (unsigned)ctas_per_head);   // query head
    const int bx = (int)(blockIdx.x % (unsigned)ctas_per_head);
    // key/value head read by query head bh: h_kv = h / (H / H_kv)
    const int b = bh / H, h_kv = (bh % H) / (H / H_kv), bh_kv = b * H_kv + h_kv;
    // Q blocks and key tiles of this sequence (a packed batch has its own per sequence;
    // Tq stays the row stride of qbar and dS)
    const SeqRange sq = seq_range(cu_q, b, n_q_max, total_q), sk = seq_range(cu_kv, b, n_kv_max, total_kv);
    const int Tq_s = cu_q ? (sq.n + kTile - 1) / kTile : Tq;
    const int Tk_s = cu_kv ? (sk.n + kTile - 1) / kTile : Tk;
    if (cu_q) causal_off = sk.n - sq.n;
    const int jt0 = bx * tiles_per_cta;
    const int n_kt = min(tiles_per_cta, Tk_s - jt0);
    if (n_kt <= 0 || Tq_s <= 0) return;  // past the end of a shorter packed sequence
    const bool is_bf16 = bf16 != 0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.bar_kfull[i], 1);
            mbar_init(&sm.bar_kempty[i], 1);
            mbar_init(&sm.bar_afull[i], 1);
            mbar_init(&sm.bar_aempty[i], 128);
            mbar_init(&sm.bar_stage_full[i], 128);
            mbar_init(&sm.bar_stage_free[i], 1);
        }
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) { tmem_alloc(&sm.tmem_base, 512); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    volatile int *abort_flag = &sm.abort_flag;

    int g = 0;              // key tiles of earlier block chunks (buffer phases run on across chunks)
    uint32_t n_chunks = 0;  // epilogue store boxes issued (staging buffer parity)
    for (int tc = 0; tc < Tq_s; tc += kDsMaxN) {
        const int nt = min(kDsMaxN, Tq_s - tc);
        const int N = (nt + 15) / 16 * 16;
        // --- stage qbar[tc .. tc + N) as hi / lo 16-bit K-major operands (128-byte swizzle)
        const float *qsrc = qbar + ((size_t)bh * Tq + tc) * D;
#pragma unroll 4
        for (int idx = threadIdx.x; idx < N * (D / 8); idx += kDsThreads) {
            const int n = idx / (D / 8), c8 = idx % (D / 8);
            float v[8];
            if (n < nt) {
                const float4 x0 = __ldg(reinterpret_cast<const float4 *>(qsrc + (size_t)n * D + c8 * 8));
                const float4 x1 = __ldg(reinterpret_cast<const float4 *>(qsrc + (size_t)n * D + c8 * 8 + 4));
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

        if (warp == 0 && lane == 0) {
            // ------------------------------ K producer ------------------------------
            int issued = 0;
            for (int i = 0; i < n_kt; ++i) {
                const int gi = g + i, buf = gi & 1;
                if (gi >= 2 && !mbar_wait(&sm.bar_kempty[buf], ((gi >> 1) & 1) ^ 1, abort_flag, status, 23)) break;
                const int j0 = (jt0 + i) * kTile;
                mbar_arrive_expect_tx(&sm.bar_kfull[buf], KA * kTile * 128);
                for (int a = 0; a < KA; ++a) {
                    if (cu_kv) tma_load_4d(sm.k[buf][a], &tm_k, &sm.bar_kfull[buf], a * 64, h_kv, sk.off + j0, 0);
                    else if (nhd) tma_load_4d(sm.k[buf][a], &tm_k, &sm.bar_kfull[buf], a * 64, h_kv, j0, b);
                    else tma_load_3d(sm.k[buf][a], &tm_k, &sm.bar_kfull[buf], a * 64, j0, bh_kv);
                }
                issued = i + 1;
            }
            if (*abort_flag)  // let the copies in flight land before the CTA exits
                for (int i = max(0, issued - 2); i < issued; ++i)
                    mbar_wait_quiet(&sm.bar_kfull[(g + i) & 1], ((g + i) >> 1) & 1, kDsDrainNs);
        } else if (warp == 1 && lane == 0) {
            // ------------------------------ MMA issuer ------------------------------
            const uint32_t idesc = idesc_f16_f32(128, N, is_bf16);
            for (int i = 0; i < n_kt; ++i) {
                const int gi = g + i, buf = gi & 1;
                if (!mbar_wait(&sm.bar_kfull[buf], (gi >> 1) & 1, abort_flag, status, 21)) break;
                if (gi >= 2 && !mbar_wait(&sm.bar_aempty[buf], ((gi >> 1) & 1) ^ 1, abort_flag, status, 24)) break;
                tc_fence_after();
                const uint32_t acc = tmem + (uint32_t)buf * 256u;
                int step = 0;
#pragma unroll
                for (int a = 0; a < KA; ++a) {
                    const uint64_t ad = smem_desc(smem_u32(sm.k[buf][a]), 1024u, 2u);
                    const uint64_t bh_d = smem_desc(smem_u32(sm.qhi[a]), 1024u, 2u);
                    const uint64_t bl_d = smem_desc(smem_u32(sm.qlo[a]), 1024u, 2u);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk, ++step) {
                        mma_f16_ss(acc, ad + 2 * kk, bh_d + 2 * kk, idesc, step > 0 ? 1u : 0u);
                        mma_f16_ss(acc, ad + 2 * kk, bl_d + 2 * kk, idesc, 1u);
                    }
                }
                mma_commit(&sm.bar_kempty[buf]);
                mma_commit(&sm.bar_afull[buf]);
            }
        } else if (warp >= 4) {
            // ------------------------------ epilogue ------------------------------
            // Store box n goes through staging buffer n & 1: its 128 writers arrive on
            // stage_full, thread 0 then issues the TMA store and, once the store before
            // it has finished reading shared memory, frees that buffer (stage_free).
            const int wq = warp & 3, et = threadIdx.x - 128;
            bool ok = true;
            for (int i = 0; ok && i < n_kt; ++i) {
                const int gi = g + i, buf = gi & 1;
                ok = __all_sync(0xFFFFFFFFu, mbar_wait(&sm.bar_afull[buf], (gi >> 1) & 1, abort_flag, status, 22));
                if (!ok) break;
                tc_fence_after();
                const int jt = jt0 + i;
                int t_lo = 0;  // Q blocks below t_lo never see key tile jt (causal)
                if (causal_skip) {
                    const int num = jt * kTile - causal_off - (kTile - 1);
                    t_lo = num <= 0 ? 0 : (num + kTile - 1) / kTile;
                }
                const uint32_t acc = tmem + (uint32_t)buf * 256u + ((uint32_t)(wq * 32) << 16);
                for (int c0 = 0; c0 < N; c0 += kDsChunk) {
                    if (tc + c0 + kDsChunk - 1 < t_lo) continue;
                    const uint32_t n = n_chunks++, sb = n & 1u;
                    uint32_t v[32];
                    tmem_ld32(acc + c0, v);
                    tmem_wait_ld_regs(v);
                    if (n >= 2) {
                        ok = __all_sync(0xFFFFFFFFu, mbar_wait(&sm.bar_stage_free[sb], ((n >> 1) - 1) & 1, abort_flag,
                                                               status, 25));
                        if (!ok) break;
                    }
                    // key k = 32 wq + lane of the tile goes to its storage position
                    const int key = wq * 32 + lane;
                    float *col = &sm.stage[sb][0][(key & 1) * (kTile / 2) + (key >> 1)];
#pragma unroll
                    for (int e = 0; e < 32; ++e) col[e * kTile] = __uint_as_float(v[e]);
                    fence_proxy_async_smem();
                    mbar_arrive(&sm.bar_stage_full[sb]);
                    if (et == 0) {
                        if (!mbar_wait(&sm.bar_stage_full[sb], (n >> 1) & 1, abort_flag, status, 26)) { ok = false; }
                        else {
                            tma_store_3d(&tm_ds, sm.stage[sb], jt * kTile, tc + c0, bh);
                            bulk_commit_group();
                            if (n >= 1) {  // box n - 1 has been read out of stage[sb ^ 1]
                                bulk_wait_group_read<1>();
                                mbar_arrive(&sm.bar_stage_free[sb ^ 1u]);
                            }
                        }
                    }
                    ok = __all_sync(0xFFFFFFFFu, ok);
                    if (!ok) break;
                }
                tc_fence_before();
                mbar_arrive(&sm.bar_aempty[buf]);
            }
            if (et == 0) bulk_wait_group<0>();
        }
        g += n_kt;
        tc_fence_before();
        __syncthreads();  // every role is done with this block chunk before qbar is restaged
        tc_fence_after();
        if (*abort_flag) break;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) { __syncwarp(); tc_fence_after(); tmem_dealloc(tmem, 512); }
}

cudaError_t launch_ds_gemm(const CUtensorMap &tm_k, const CUtensorMap &tm_ds, const float *qbar, const Shape &s,
                           int nhd, int bf16, int causal_skip, int causal_off, const int *cu_q, const int *cu_kv,
                           int *status, cudaStream_t stream) {
    // Key tiles per CTA: 16 (the staged qbar is reused across them), or fewer when the
    // grid would otherwise leave SMs idle (short sequences): about two CTAs per SM.
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long units = (long long)s.BH * s.Tk;
    int tpc = (int)((units + 2LL * sms - 1) / (2LL * sms));
    tpc = tpc < 1 ? 1 : (tpc > kDsTilesPerCta ? kDsTilesPerCta : tpc);
    const int ctas_per_head = (s.Tk + tpc - 1) / tpc;
    const unsigned grid = (unsigned)((size_t)ctas_per_head * s.BH);
    if (s.d == 128) {
        const size_t smem = sizeof(DsSmem<128>) + 1024;
        cudaError_t e = cudaFuncSetAttribute(ds_gemm_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        ds_gemm_kernel<128><<<grid, kDsThreads, smem, stream>>>(tm_k, tm_ds, qbar, s.H, s.H_kv, s.Tq, s.Tk, nhd, bf16,
                                                                 causal_skip, causal_off, cu_q, cu_kv, s.n_q, s.n_kv,
                                                                 s.total_q, s.total_kv, tpc, ctas_per_head, status);
    } else {
        const size_t smem = sizeof(DsSmem<64>) + 1024;
        cudaError_t e = cudaFuncSetAttribute(ds_gemm_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        ds_gemm_kernel<64><<<grid, kDsThreads, smem, stream>>>(tm_k, tm_ds, qbar, s.H, s.H_kv, s.Tq, s.Tk, nhd, bf16,
                                                                causal_skip, causal_off, cu_q, cu_kv, s.n_q, s.n_kv,
                                                                s.total_q, s.total_kv, tpc, ctas_per_head, status);
    }
    return cudaGetLastError();
}

}  // namespace sage
