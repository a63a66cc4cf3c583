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
// previous one).  The epilogue threads (one per key) store their accumulator rows
// straight to dS[block][position], keys of each 128-key tile in the storage order
// (even, then odd): for one block a warp's 32 keys are two runs of 16 consecutive
// positions.  32-block chunks whose blocks can never see a key tile (causal) are not
// written.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "sage_device.cuh"
#include "sage_internal.h"

namespace sage {

constexpr int kDsThreads = 256;
constexpr int kDsMaxN = 256;
constexpr int kDsChunk = 32;   // Q blocks per tensor-memory load of the epilogue
constexpr uint64_t kDsDrainNs = 50ull * 1000ull * 1000ull;

// Roles (256 threads): warp 0 loads K tiles (TMA, two buffers); warp 1 issues the
// MMAs into one of two 256-column tensor-memory accumulators, so the product of
// key tile i + 1 overlaps the epilogue of tile i; warps 4-7 (one per lane
// quadrant) load each 32-block chunk of D[key][block] and store it to dS.  All 256
// threads stage qbar.  One CTA per SM: it holds all 512 tensor-memory columns.
template <int D>
struct __align__(1024) DsSmem {
    static constexpr int KA = D / 64;              // 128-byte (64-element) atoms along d
    uint8_t qhi[KA][kDsMaxN * 128];
    uint8_t qlo[KA][kDsMaxN * 128];
    uint8_t k[2][KA][kTile * 128];
    uint64_t bar_kfull[2], bar_kempty[2], bar_afull[2], bar_aempty[2];
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
    ds_gemm_kernel(const __grid_constant__ CUtensorMap tm_k, float *__restrict__ ds_out, const float *__restrict__ qbar,
                   int BH, int H, int H_kv, int Tq, int Tk, int nhd, int bf16, int causal_skip, int causal_off,
                   const int *__restrict__ cu_q, const int *__restrict__ cu_kv, int n_q_max, int n_kv_max, int total_q,
                   int total_kv, int *status) {
    constexpr int KA = D / 64;
    extern __shared__ uint8_t smem_raw[];
    DsSmem<D> &sm = *reinterpret_cast<DsSmem<D> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // Persistent CTAs: this CTA's work is one contiguous range of the (query head, key
    // tile) units in head-major order, the ranges of the grid balanced to one unit.
    const long long n_units = (long long)BH * Tk;
    const long long u_lo = n_units * blockIdx.x / gridDim.x, u_hi = n_units * (blockIdx.x + 1) / gridDim.x;
    const bool is_bf16 = bf16 != 0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.bar_kfull[i], 1);
            mbar_init(&sm.bar_kempty[i], 1);
            mbar_init(&sm.bar_afull[i], 1);
            mbar_init(&sm.bar_aempty[i], 128);
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

    int g = 0;   // key tiles of earlier block chunks and heads (buffer phases run on across them)
    for (long long u = u_lo; u < u_hi;) {
        // the next run of key tiles [jt0, jt0 + n_kt) of one query head bh
        const int bh = (int)(u / Tk), jt0 = (int)(u % Tk);
        const int jt_end = (int)min((long long)Tk, jt0 + (u_hi - u));
        u += jt_end - jt0;
        // key/value head read by query head bh: h_kv = h / (H / H_kv)
        const int b = bh / H, h_kv = (bh % H) / (H / H_kv), bh_kv = b * H_kv + h_kv;
        // Q blocks and key tiles of this sequence (a packed batch has its own per
        // sequence; Tq stays the row stride of qbar and dS)
        const SeqRange sq = seq_range(cu_q, b, n_q_max, total_q), sk = seq_range(cu_kv, b, n_kv_max, total_kv);
        const int Tq_s = cu_q ? (sq.n + kTile - 1) / kTile : Tq;
        const int Tk_s = cu_kv ? (sk.n + kTile - 1) / kTile : Tk;
        const int c_off = cu_q ? sk.n - sq.n : causal_off;
        const int n_kt = min(jt_end, Tk_s) - jt0;
        if (n_kt <= 0 || Tq_s <= 0) continue;  // past the end of a shorter packed sequence
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
                // dS of this head is [Tq][Tk * 128]; rows (blocks) past Tq are not written
                const int wq = warp & 3;
                const int key = wq * 32 + lane;   // this thread's tensor-memory lane
                const size_t row_stride = (size_t)Tk * kTile;
                bool ok = true;
                for (int i = 0; ok && i < n_kt; ++i) {
                    const int gi = g + i, buf = gi & 1;
                    ok = __all_sync(0xFFFFFFFFu, mbar_wait(&sm.bar_afull[buf], (gi >> 1) & 1, abort_flag, status, 22));
                    if (!ok) break;
                    tc_fence_after();
                    const int jt = jt0 + i;
                    int t_lo = 0;  // Q blocks below t_lo never see key tile jt (causal)
                    if (causal_skip) {
                        const int num = jt * kTile - c_off - (kTile - 1);
                        t_lo = num <= 0 ? 0 : (num + kTile - 1) / kTile;
                    }
                    const uint32_t acc = tmem + (uint32_t)buf * 256u + ((uint32_t)(wq * 32) << 16);
                    float *dst = ds_out + ((size_t)bh * Tq + tc) * row_stride + (size_t)jt * kTile +
                                 (key & 1) * (kTile / 2) + (key >> 1);
                    for (int c0 = 0; c0 < N; c0 += kDsChunk) {
                        if (tc + c0 + kDsChunk - 1 < t_lo) continue;
                        uint32_t v[32];
                        tmem_ld32(acc + c0, v);
                        tmem_wait_ld_regs(v);
                        const int e_max = min(kDsChunk, Tq - (tc + c0));
                        if (e_max >= kDsChunk) {
#pragma unroll
                            for (int e = 0; e < kDsChunk; ++e) dst[(size_t)(c0 + e) * row_stride] = __uint_as_float(v[e]);
                        } else {
#pragma unroll
                            for (int e = 0; e < kDsChunk; ++e)
                                if (e < e_max) dst[(size_t)(c0 + e) * row_stride] = __uint_as_float(v[e]);
                        }
                    }
                    tc_fence_before();
                    mbar_arrive(&sm.bar_aempty[buf]);
                }
            }
            g += n_kt;
            tc_fence_before();
            __syncthreads();  // every role is done with this block chunk before qbar is restaged
            tc_fence_after();
            if (*abort_flag) break;
        }
        if (*abort_flag) break;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) { __syncwarp(); tc_fence_after(); tmem_dealloc(tmem, 512); }
}

// Dynamic shared memory of a CTA: its layout (plus alignment slack), and at least
// 120 KB, so that no two CTAs share an SM (each allocates all 512 tensor-memory
// columns).
static size_t ds_smem_bytes(size_t layout_bytes) {
    const size_t b = layout_bytes + 1024;
    return b < 120u * 1024u ? 120u * 1024u : b;
}

cudaError_t launch_ds_gemm(const CUtensorMap &tm_k, float *ds_out, const float *qbar, const Shape &s,
                           int nhd, int bf16, int causal_skip, int causal_off, const int *cu_q, const int *cu_kv,
                           int *status, cudaStream_t stream) {
    // One persistent CTA per SM (or per unit, if fewer)
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long units = (long long)s.BH * s.Tk;
    const unsigned grid = (unsigned)(units < sms ? units : sms);
    if (grid == 0) return cudaSuccess;
    if (s.d == 128) {
        const size_t smem = ds_smem_bytes(sizeof(DsSmem<128>));
        cudaError_t e = cudaFuncSetAttribute(ds_gemm_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        ds_gemm_kernel<128><<<grid, kDsThreads, smem, stream>>>(tm_k, ds_out, qbar, s.BH, s.H, s.H_kv, s.Tq, s.Tk, nhd, bf16,
                                                                 causal_skip, causal_off, cu_q, cu_kv, s.n_q, s.n_kv,
                                                                 s.total_q, s.total_kv, status);
    } else {
        const size_t smem = ds_smem_bytes(sizeof(DsSmem<64>));
        cudaError_t e = cudaFuncSetAttribute(ds_gemm_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        ds_gemm_kernel<64><<<grid, kDsThreads, smem, stream>>>(tm_k, ds_out, qbar, s.BH, s.H, s.H_kv, s.Tq, s.Tk, nhd, bf16,
                                                                causal_skip, causal_off, cu_q, cu_kv, s.n_q, s.n_kv,
                                                                s.total_q, s.total_kv, status);
    }
    return cudaGetLastError();
}

}  // namespace sage
