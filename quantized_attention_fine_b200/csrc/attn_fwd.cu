// attn_fwd.cu -- fused sm_100a attention kernel of the smoothed-INT8-QK / FP8-PV
// forward, plus two diagnostic kernels that reuse its MMA issue code.
//
// Method (SageAttention2, arXiv 2411.10958, abstract; SageAttention2++ verdict on
// pith.science, key_machinery): S = dQ(i) dK(j) (Q_int . K_int) + dS[t, j] on the
// INT8 tensor core; tiled online softmax ("Online normalizer calculation for
// softmax", Milakov and Gimelshein) over 128-key tiles; P~ = exp(x - m) scaled by
// Pr and rounded to E4M3; O += P8 . V8 on the FP8 tensor core, FP32 accumulation
// in tensor memory; O = acc * delta_V / (Pr l).
//
// One CTA computes one 128-row Q tile of one head (192 threads):
//   warps 0-3  softmax + epilogue; thread i owns query row i = tensor-memory lane i
//   warp 4     TMA producer: Q tile once, then K / V^T tiles, dS and delta_K runs
//              through a 3-stage shared-memory ring
//   warp 5     tensor-memory allocation and single-thread tcgen05.mma issue
// Tensor memory (512 columns): S double buffer (int32, columns 0-127 and 128-255),
// O accumulator (fp32, columns 256 .. 256 + d).  QK^T of tile j + 1 runs on the
// tensor core while the softmax warps work on tile j.
// Every wait is bounded: a wait that runs out records SAGE_ERR_TIMEOUT in the
// status block, raises a CTA-wide abort flag that makes every role leave its loop,
// drains the copies in flight, frees tensor memory and exits.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "sage_device.cuh"
#include "sage_internal.h"

namespace sage {

constexpr int kStages = 3;
constexpr int kAttnThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 256;
constexpr uint64_t kDrainNs = 50ull * 1000ull * 1000ull;

// Wait-site ids recorded with a timeout.
enum { kSiteQ = 1, kSiteFull = 2, kSiteEmpty = 3, kSiteS = 4, kSiteP = 5, kSiteO = 6, kSiteDebug = 9 };

template <int D>
struct __align__(1024) AttnSmem {
    uint8_t q[kTile * D];
    uint8_t k[kStages][kTile * D];
    uint8_t v[kStages][D * kTile];
    uint8_t p[kTile * kTile];
    float ds[kStages][kTile];
    float dk[kStages][kTile / kKeyRun];
    uint64_t bar_q, bar_full[kStages], bar_empty[kStages], bar_s[2], bar_p, bar_o, bar_drain;
    uint32_t tmem_base;
    int abort_flag;
};

// K-major operand layout of a Q or K tile: rows of d bytes; d = 128 uses the
// 128-byte swizzle (8-row groups 1024 bytes apart), d = 64 the 64-byte swizzle.
template <int D>
struct QkLayout {
    static constexpr uint32_t layout = (D == 128) ? 2u : 4u;
    static constexpr uint32_t sbo = (D == 128) ? 1024u : 512u;
};

// S[d_tmem] = Q_tile . K_tile^T: d / 32 tcgen05.mma kind::i8 (M = 128, N = 128,
// K = 32 each), the descriptor start advancing 32 bytes along the swizzled row.
template <int D>
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint32_t q_saddr, uint32_t k_saddr) {
    constexpr uint32_t idesc = idesc_s8_s32(128, 128);
#pragma unroll
    for (int kk = 0; kk < D / 32; ++kk) {
        const uint64_t a = smem_desc(q_saddr + kk * 32, QkLayout<D>::sbo, QkLayout<D>::layout);
        const uint64_t b = smem_desc(k_saddr + kk * 32, QkLayout<D>::sbo, QkLayout<D>::layout);
        mma_s8_ss(d_tmem, a, b, idesc, kk > 0 ? 1u : 0u);
    }
}

// O[d_tmem] (+)= P_tile . V_tile: P is 128 rows x 128 keys (E4M3, 128-byte rows,
// 128-byte swizzle), V^T is d rows x 128 keys (same layout); 4 tcgen05.mma
// kind::f8f6f4 with M = 128, N = d, K = 32.
template <int D>
__device__ __forceinline__ void issue_pv(uint32_t d_tmem, uint32_t p_saddr, uint32_t v_saddr, bool accumulate) {
    constexpr uint32_t idesc = idesc_e4m3_f32(128, D);
#pragma unroll
    for (int kk = 0; kk < kTile / 32; ++kk) {
        const uint64_t a = smem_desc(p_saddr + kk * 32, 1024u, 2u);
        const uint64_t b = smem_desc(v_saddr + kk * 32, 1024u, 2u);
        mma_e4m3_ss(d_tmem, a, b, idesc, (accumulate || kk > 0) ? 1u : 0u);
    }
}

// A bounded wait whose outcome is the same for all 32 lanes (so that the warp
// leaves its loop together and its .sync.aligned instructions stay converged).
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag, int *status,
                                          int site) {
    const bool ok = mbar_wait(bar, parity, abort_flag, status, site);
    return __all_sync(0xFFFFFFFFu, ok);
}

__device__ __forceinline__ void store_row_chunk(void *dst, const float (&y)[32], int out_bf16) {
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        if (out_bf16) {
            __nv_bfloat162 h = __floats2bfloat162_rn(y[2 * i], y[2 * i + 1]);
            w[i] = *reinterpret_cast<uint32_t *>(&h);
        } else {
            __half2 h = __floats2half2_rn(y[2 * i], y[2 * i + 1]);
            w[i] = *reinterpret_cast<uint32_t *>(&h);
        }
    }
    uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
    for (int i = 0; i < 4; ++i) d4[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
}

template <int D>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ AttnParams p) {
    extern __shared__ uint8_t smem_raw[];
    AttnSmem<D> &sm =
        *reinterpret_cast<AttnSmem<D> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // Work item: longest Q tiles first when causal.
    const int t_idx = blockIdx.x / p.BH;
    const int bh = blockIdx.x % p.BH;
    const int t = p.causal ? (p.Tq - 1 - t_idx) : t_idx;
    const int b = bh / p.H, h = bh % p.H;
    const int off = p.n_kv - p.n_q;
    int n_tiles = p.Tk;
    if (p.causal) {
        const int last_key = min(t * kTile + kTile - 1, p.n_q - 1) + off;
        n_tiles = last_key < 0 ? 0 : min(p.Tk, last_key / kTile + 1);
    }
    const int64_t o_base = (int64_t)b * p.so_b + (int64_t)h * p.so_h;

    if (n_tiles == 0) {  // no row of this tile sees any key: O = 0
        if (warp < 4) {
            const int row = t * kTile + warp * 32 + lane;
            if (row < p.n_q) {
                uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.o) + o_base + (int64_t)row * p.so_n);
#pragma unroll
                for (int i = 0; i < D / 8; ++i) dst[i] = make_uint4(0, 0, 0, 0);
            }
        }
        return;
    }

    if (threadIdx.x == 0) {
        mbar_init(&sm.bar_q, 1);
        for (int s = 0; s < kStages; ++s) { mbar_init(&sm.bar_full[s], 1); mbar_init(&sm.bar_empty[s], 1); }
        mbar_init(&sm.bar_s[0], 1);
        mbar_init(&sm.bar_s[1], 1);
        mbar_init(&sm.bar_p, 128);
        mbar_init(&sm.bar_o, 1);
        mbar_init(&sm.bar_drain, 1);
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 5) {
        tmem_alloc(&sm.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    volatile int *abort_flag = &sm.abort_flag;

    if (warp == 4) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_v);
            mbar_arrive_expect_tx(&sm.bar_q, kTile * D);
            tma_load_2d(sm.q, &tm_q, &sm.bar_q, 0, bh * p.nq_pad + t * kTile);
            const uint32_t stage_bytes = kTile * D * 2 + (p.use_ds ? kTile * 4 : 0) + (kTile / kKeyRun) * 4;
            const float *ds_row = p.ds + ((size_t)bh * p.Tq + t) * p.nk_pad;
            const float *dk_row = p.dk + (size_t)bh * (p.nk_pad / kKeyRun);
            int issued = 0;
            for (int it = 0; it < n_tiles; ++it) {
                const int s = it % kStages;
                if (it >= kStages && !mbar_wait(&sm.bar_empty[s], ((it / kStages) & 1) ^ 1, abort_flag, p.status, kSiteEmpty))
                    break;
                issued = it + 1;
                if (p.fault_inject && it == 0) continue;  // diagnostic: leave stage 0 unsignalled
                mbar_arrive_expect_tx(&sm.bar_full[s], stage_bytes);
                tma_load_2d(sm.k[s], &tm_k, &sm.bar_full[s], 0, bh * p.nk_pad + it * kTile);
                tma_load_2d(sm.v[s], &tm_v, &sm.bar_full[s], it * kTile, bh * D);
                if (p.use_ds) bulk_load(sm.ds[s], ds_row + it * kTile, kTile * 4, &sm.bar_full[s]);
                bulk_load(sm.dk[s], dk_row + it * (kTile / kKeyRun), (kTile / kKeyRun) * 4, &sm.bar_full[s]);
            }
            if (*abort_flag) {  // let the copies in flight land before the CTA exits
                mbar_wait_quiet(&sm.bar_q, 0, kDrainNs);
                for (int it = max(0, issued - kStages); it < issued; ++it) {
                    if (p.fault_inject && it == 0) continue;
                    mbar_wait_quiet(&sm.bar_full[it % kStages], (it / kStages) & 1, kDrainNs);
                }
            }
        }
    } else if (warp == 5) {
        // ------------------------------ MMA issuer ------------------------------
        if (lane == 0) {
            const uint32_t q_s = smem_u32(sm.q), p_s = smem_u32(sm.p);
            bool ok = mbar_wait(&sm.bar_q, 0, abort_flag, p.status, kSiteQ);
            auto qk = [&](int i) -> bool {
                const int s = i % kStages;
                if (!mbar_wait(&sm.bar_full[s], (i / kStages) & 1, abort_flag, p.status, kSiteFull)) return false;
                tc_fence_after();
                issue_qk<D>(tmem + (uint32_t)(i & 1) * 128u, q_s, smem_u32(sm.k[s]));
                mma_commit(&sm.bar_s[i & 1]);
                return true;
            };
            if (ok) ok = qk(0);
            for (int it = 0; ok && it < n_tiles; ++it) {
                if (it + 1 < n_tiles && !qk(it + 1)) break;
                if (!mbar_wait(&sm.bar_p, it & 1, abort_flag, p.status, kSiteP)) break;
                tc_fence_after();
                const int s = it % kStages;
                issue_pv<D>(tmem + kTmemO, p_s, smem_u32(sm.v[s]), it > 0);
                mma_commit(&sm.bar_o);
                mma_commit(&sm.bar_empty[s]);
            }
            mma_commit(&sm.bar_drain);
            mbar_wait_quiet(&sm.bar_drain, 0, kDrainNs);
        }
    } else {
        // ------------------------- softmax (warps 0-3) -------------------------
        const int r = warp * 32 + lane;
        const int row = t * kTile + r;
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        const float dq = p.dq[(size_t)bh * p.nq_pad + row];
        const float c = p.scale_log2;
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        for (int it = 0; it < n_tiles; ++it) {
            const int s = it % kStages;
            if (!warp_wait(&sm.bar_s[it & 1], (it >> 1) & 1, abort_flag, p.status, kSiteS)) { ok = false; break; }
            if (!warp_wait(&sm.bar_full[s], (it / kStages) & 1, abort_flag, p.status, kSiteFull)) { ok = false; break; }
            tc_fence_after();
            uint32_t sv[4][32];
            const uint32_t s_addr = tmem + lane_base + (uint32_t)(it & 1) * 128u;
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) tmem_ld32(s_addr + q4 * 32, sv[q4]);
            tmem_wait_ld_regs(sv[0]);
            reg_fence(sv[1]);
            reg_fence(sv[2]);
            reg_fence(sv[3]);

            float a[kTile / kKeyRun];
#pragma unroll
            for (int g = 0; g < kTile / kKeyRun; ++g) a[g] = dq * sm.dk[s][g];
            const bool masked = (it * kTile + kTile > p.n_kv) || (p.causal && it * kTile + kTile - 1 > t * kTile + off);
            float tmax = -INFINITY;
#pragma unroll
            for (int j = 0; j < kTile; ++j) {
                const float ds = p.use_ds ? sm.ds[s][j] : 0.f;
                float x = fmaf((float)(int)sv[j / 32][j % 32], a[j / kKeyRun], ds);
                if (masked) {
                    const int key = it * kTile + j;
                    const bool vis = key < p.n_kv && (!p.causal || key <= row + off);
                    x = vis ? x : -INFINITY;
                }
                sv[j / 32][j % 32] = __float_as_uint(x);
                tmax = fmaxf(tmax, x);
            }
            const float m_new = fmaxf(m, tmax);
            float alpha, bias;
            if (m_new == -INFINITY) {
                alpha = 1.f;
                bias = 0.f;
            } else {
                alpha = ex2_approx((m - m_new) * c);
                bias = p.log2_pr - m_new * c;
            }
            float sum = 0.f;
            uint32_t pk[kTile / 4];
#pragma unroll
            for (int j = 0; j < kTile; j += 4) {
                float e[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) e[u] = ex2_approx(fmaf(__uint_as_float(sv[(j + u) / 32][(j + u) % 32]), c, bias));
                sum += (e[0] + e[1]) + (e[2] + e[3]);
                pk[j / 4] = pack_e4m3x4(e[0], e[1], e[2], e[3]);
            }
            l = l * alpha + sum;
            const bool rescale = (it > 0) && (alpha != 1.f);
            m = m_new;

            if (it > 0) {  // PV of the previous tile must be done before P and O are touched
                if (!warp_wait(&sm.bar_o, (it - 1) & 1, abort_flag, p.status, kSiteO)) { ok = false; break; }
                tc_fence_after();
            }
#pragma unroll
            for (int c16 = 0; c16 < 8; ++c16)
                *reinterpret_cast<uint4 *>(sm.p + sw128_offset(r, c16)) =
                    make_uint4(pk[4 * c16], pk[4 * c16 + 1], pk[4 * c16 + 2], pk[4 * c16 + 3]);
            if (__any_sync(0xFFFFFFFFu, rescale)) {
#pragma unroll
                for (int c0 = 0; c0 < D; c0 += 32) {
                    uint32_t ov[32];
                    tmem_ld32(tmem + lane_base + kTmemO + c0, ov);
                    tmem_wait_ld_regs(ov);
#pragma unroll
                    for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
                    tmem_st32(tmem + lane_base + kTmemO + c0, ov);
                }
                tmem_wait_st();
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&sm.bar_p);
        }
        if (ok) ok = warp_wait(&sm.bar_o, (n_tiles - 1) & 1, abort_flag, p.status, kSiteO);
        if (ok) {
            tc_fence_after();
            const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
            const float *dv = p.dv + (size_t)bh * D;
            uint16_t *orow = static_cast<uint16_t *>(p.o) + o_base + (int64_t)row * p.so_n;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t ov[32];
                tmem_ld32(tmem + lane_base + kTmemO + c0, ov);
                tmem_wait_ld_regs(ov);
                float y[32];
#pragma unroll
                for (int i = 0; i < 32; i += 4) {
                    const float4 s4 = __ldg(reinterpret_cast<const float4 *>(dv + c0 + i));
                    y[i] = __uint_as_float(ov[i]) * s4.x * inv_l;
                    y[i + 1] = __uint_as_float(ov[i + 1]) * s4.y * inv_l;
                    y[i + 2] = __uint_as_float(ov[i + 2]) * s4.z * inv_l;
                    y[i + 3] = __uint_as_float(ov[i + 3]) * s4.w * inv_l;
                }
                if (row < p.n_q) store_row_chunk(orow + c0, y, p.out_bf16);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int D>
static cudaError_t launch_attention_d(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                      const AttnParams &p, cudaStream_t stream) {
    const size_t smem = sizeof(AttnSmem<D>) + 1024;
    cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)p.Tq * (unsigned)p.BH;
    attn_fwd_kernel<D><<<grid, kAttnThreads, smem, stream>>>(tq, tk, tv, p);
    return cudaGetLastError();
}

cudaError_t launch_attention(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                             const AttnParams &p, int d, cudaStream_t stream) {
    if (d == 128) return launch_attention_d<128>(tq, tk, tv, p, stream);
    return launch_attention_d<64>(tq, tk, tv, p, stream);
}

// ---------------------------------------------------------------------------
// Diagnostic: one S tile straight from tensor memory.
// ---------------------------------------------------------------------------
template <int D>
struct __align__(1024) QkDebugSmem {
    uint8_t q[kTile * D];
    uint8_t k[kTile * D];
    uint64_t bar_ld, bar_mma;
    uint32_t tmem_base;
    int abort_flag;
};

template <int D>
__global__ void __launch_bounds__(128, 1)
    debug_qk_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k, int q_row0,
                    int k_row0, int32_t *out, int *status) {
    extern __shared__ uint8_t smem_raw[];
    QkDebugSmem<D> &sm =
        *reinterpret_cast<QkDebugSmem<D> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(&sm.bar_ld, 1);
        mbar_init(&sm.bar_mma, 1);
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) { tmem_alloc(&sm.tmem_base, 128); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    volatile int *abort_flag = &sm.abort_flag;
    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(&sm.bar_ld, 2 * kTile * D);
        tma_load_2d(sm.q, &tm_q, &sm.bar_ld, 0, q_row0);
        tma_load_2d(sm.k, &tm_k, &sm.bar_ld, 0, k_row0);
        if (mbar_wait(&sm.bar_ld, 0, abort_flag, status, kSiteDebug)) {
            tc_fence_after();
            issue_qk<D>(tmem, smem_u32(sm.q), smem_u32(sm.k));
        } else {
            mbar_wait_quiet(&sm.bar_ld, 0, kDrainNs);
        }
        mma_commit(&sm.bar_mma);
    }
    __syncwarp();
    mbar_wait(&sm.bar_mma, 0, abort_flag, status, kSiteDebug);
    tc_fence_after();
    __syncthreads();
    if (*abort_flag == 0) {
        const int r = warp * 32 + lane;
#pragma unroll
        for (int c0 = 0; c0 < kTile; c0 += 32) {
            uint32_t v[32];
            tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + c0, v);
            tmem_wait_ld_regs(v);
            int4 *dst = reinterpret_cast<int4 *>(out + (size_t)r * kTile + c0);
#pragma unroll
            for (int i = 0; i < 8; ++i) dst[i] = make_int4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) { __syncwarp(); tc_fence_after(); tmem_dealloc(tmem, 128); }
}

cudaError_t launch_debug_qk_tile(const CUtensorMap &tq, const CUtensorMap &tk, int d, int q_row0, int k_row0,
                                 int32_t *s_out, int *status, cudaStream_t stream) {
    if (d == 128) {
        const size_t smem = sizeof(QkDebugSmem<128>) + 1024;
        cudaError_t e = cudaFuncSetAttribute(debug_qk_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        debug_qk_kernel<128><<<1, 128, smem, stream>>>(tq, tk, q_row0, k_row0, s_out, status);
    } else {
        const size_t smem = sizeof(QkDebugSmem<64>) + 1024;
        cudaError_t e = cudaFuncSetAttribute(debug_qk_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        debug_qk_kernel<64><<<1, 128, smem, stream>>>(tq, tk, q_row0, k_row0, s_out, status);
    }
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Diagnostic: sum over tiles of P . V on the FP8 path, one FP32 accumulator.
// P and V^T tiles are copied row by row into the 128-byte-swizzled layout the
// attention kernel uses for P.
// ---------------------------------------------------------------------------
template <int D>
struct __align__(1024) PvDebugSmem {
    uint8_t p[kTile * kTile];
    uint8_t v[D * kTile];
    uint64_t bar_mma;
    uint32_t tmem_base;
    int abort_flag;
};

template <int D>
__global__ void __launch_bounds__(128, 1)
    debug_pv_kernel(const uint8_t *p, const uint8_t *vt, int n_tiles, float *out, int *status) {
    extern __shared__ uint8_t smem_raw[];
    PvDebugSmem<D> &sm =
        *reinterpret_cast<PvDebugSmem<D> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = threadIdx.x;
    if (threadIdx.x == 0) {
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
    bool ok = true;
    for (int tile = 0; tile < n_tiles && ok; ++tile) {
        const uint4 *src_p = reinterpret_cast<const uint4 *>(p + ((size_t)tile * kTile + r) * kTile);
#pragma unroll
        for (int c16 = 0; c16 < 8; ++c16) *reinterpret_cast<uint4 *>(sm.p + sw128_offset(r, c16)) = src_p[c16];
        if (r < D) {
            const uint4 *src_v = reinterpret_cast<const uint4 *>(vt + ((size_t)tile * D + r) * kTile);
#pragma unroll
            for (int c16 = 0; c16 < 8; ++c16) *reinterpret_cast<uint4 *>(sm.v + sw128_offset(r, c16)) = src_v[c16];
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (threadIdx.x == 0) {
            tc_fence_after();
            issue_pv<D>(tmem, smem_u32(sm.p), smem_u32(sm.v), tile > 0);
            mma_commit(&sm.bar_mma);
        }
        __syncwarp();
        mbar_wait(&sm.bar_mma, tile & 1, abort_flag, status, kSiteDebug);
        tc_fence_after();
        __syncthreads();
        ok = (*abort_flag == 0);
    }
    if (ok && n_tiles > 0) {
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t v[32];
            tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + c0, v);
            tmem_wait_ld_regs(v);
#pragma unroll
            for (int i = 0; i < 32; ++i) out[(size_t)r * D + c0 + i] = __uint_as_float(v[i]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) { __syncwarp(); tc_fence_after(); tmem_dealloc(tmem, 256); }
}

cudaError_t launch_debug_pv(const uint8_t *p, const uint8_t *vt, int n_tiles, int d, float *o, int *status,
                            cudaStream_t stream) {
    if (d == 128) {
        const size_t smem = sizeof(PvDebugSmem<128>) + 1024;
        cudaError_t e = cudaFuncSetAttribute(debug_pv_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        debug_pv_kernel<128><<<1, 128, smem, stream>>>(p, vt, n_tiles, o, status);
    } else {
        const size_t smem = sizeof(PvDebugSmem<64>) + 1024;
        cudaError_t e = cudaFuncSetAttribute(debug_pv_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        debug_pv_kernel<64><<<1, 128, smem, stream>>>(p, vt, n_tiles, o, status);
    }
    return cudaGetLastError();
}

}  // namespace sage
