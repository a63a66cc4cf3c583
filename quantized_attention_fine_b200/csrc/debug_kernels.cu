// debug_kernels.cu -- diagnostic kernels: one QK^T tile and a PV sum through the
// attention kernel's own MMA issue sequences (attn_mma.cuh), and the throughput of
// the tcgen05.mma forms the forward uses, and of the FP8 form with an FP16 accumulator that SageAttention2++ builds
// on ("SageAttention2++" verdict on arXiv 2505.21136, key_machinery: the
// FP16-accumulator FP8 instruction, taken as twice as fast on RTX4090 / RTX5090).
//
// Each CTA (one per SM) zeroes an A tile (128 rows) and a B tile (256 rows) of
// 128-byte K-major rows in shared memory, and one thread issues n_iter MMAs of
// M = 128, N = 256 and one 32-byte K step each into a tensor-memory accumulator,
// then waits (bounded) for their completion.  The host times the launch; the MMA
// count and shape give the rate.  Kinds:
//   0  kind::f8f6f4, E4M3 x E4M3, FP32 accumulator   (the forward's PV)
//   1  kind::f8f6f4, E4M3 x E4M3, FP16 accumulator   (SageAttention2++ PV)
//   2  kind::i8, S8 x S8, S32 accumulator            (the forward's QK^T)
//   3  kind::f16, BF16 x BF16, FP32 accumulator      (dS)
#include <cuda_fp16.h>

#include "attn_mma.cuh"
#include "sage_device.cuh"
#include "sage_internal.h"

namespace sage {

namespace {

constexpr int kSiteDebug = 9;
constexpr uint64_t kDrainNs = 50ull * 1000ull * 1000ull;

struct __align__(1024) MmaRateSmem {
    uint8_t a[128 * 128];
    uint8_t b[256 * 128];
    uint64_t bar;
    uint32_t tmem_base;
    int abort_flag;
};

constexpr int kSiteRate = 41;
// Dynamic shared memory requested per CTA: large enough that one CTA runs per SM.
constexpr size_t kRateSmem = 160u * 1024u;

}  // namespace

// ---------------------------------------------------------------------------
// FP4 quantization of smoothed rows, the two-level microscaling form of 4-bit Q / K
// on B200 (block-scaled tcgen05.mma kind::mxf4nvf4; "SageAttention3: Microscaling
// FP4 Attention", listed among the notes' related papers): per 128-row tile
//   g = amax / (6 * 448)  (1 if amax = 0),
// per row and 16 channels
//   sf = E4M3(fp32(amax / g) / 6)  (1 if amax = 0; 2^-9 if it rounds to 0),
// per element
//   code = E2M1(fp32(x / fp32(g * sf)))  (round to nearest even, saturating at 6).
// One CTA per tile, 8 warps of 16 rows, lane l holding channels l*VEC ..; a 16-channel
// block spans 16 / VEC lanes.  Output: codes packed two per byte (channel 2i in the
// low nibble), [n_pad][d / 2]; E4M3 scale codes [n_pad][d / 16]; g per tile.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) debug_quant_fp4_kernel(const float *__restrict__ xs, int n_rows,
                                                              uint8_t *__restrict__ codes, uint8_t *__restrict__ sf,
                                                              float *__restrict__ g_out) {
    constexpr int VEC = D / 32, LPB = 16 / VEC;  // lanes per 16-channel block
    __shared__ float s_max[8];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r0 = blockIdx.x * kTile + warp * 16;
    float x[16][VEC];
    float am = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int r = r0 + i;
#pragma unroll
        for (int v = 0; v < VEC; ++v) {
            x[i][v] = (r < n_rows) ? xs[(size_t)r * D + lane * VEC + v] : 0.f;
            am = fmaxf(am, fabsf(x[i][v]));
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, o));
    if (lane == 0) s_max[warp] = am;
    __syncthreads();
    float tile_max = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) tile_max = fmaxf(tile_max, s_max[w]);
    const float g = (tile_max == 0.f) ? 1.f : __fdiv_rn(tile_max, 2688.f);
    if (threadIdx.x == 0) g_out[blockIdx.x] = g;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        float bm = 0.f;
#pragma unroll
        for (int v = 0; v < VEC; ++v) bm = fmaxf(bm, fabsf(x[i][v]));
#pragma unroll
        for (int o = 1; o < LPB; o <<= 1) bm = fmaxf(bm, __shfl_xor_sync(0xFFFFFFFFu, bm, o));
        uint8_t sc = 0x38;
        if (bm != 0.f) {
            sc = (uint8_t)(pack_e4m3x4(__fdiv_rn(__fdiv_rn(bm, g), 6.f), 0.f, 0.f, 0.f) & 0xFFu);
            if ((sc & 0x7F) == 0) sc = 0x01;
        }
        const float delta = __fmul_rn(g, e4m3_value(sc));
        const size_t row = (size_t)(r0 + i);
        if (lane % LPB == 0) sf[row * (D / 16) + lane / LPB] = sc;
        uint32_t packed = 0;  // VEC codes, 4 bits each, channel lane*VEC + v at bits 4v
#pragma unroll
        for (int v = 0; v < VEC; v += 2)
            packed |= e2m1x2(__fdiv_rn(x[i][v + 1], delta), __fdiv_rn(x[i][v], delta)) << (4 * v);
        uint8_t *dst = codes + row * (D / 2) + lane * (VEC / 2);
        if constexpr (VEC == 4) *reinterpret_cast<uint16_t *>(dst) = (uint16_t)packed;
        else *dst = (uint8_t)packed;
    }
}

// The pre-pass quotient routines against the IEEE division: for every finite 16-bit
// input pattern x (bf16 when `bf16`, else fp16) and every delta of the list with
// |x| <= 448 delta (the range a quantization group presents: its amax over 448 or
// 127), where the quantizers use the routines (delta >= kQuotientMinDelta):
// - quotient2_rn(x), quotient2_rn(-x) against __fdiv_rn bit for bit where the quotient
//   is at least 2^-20 (below, the quotient or the remainder may be subnormal);
// - e4m3x4_codes_rn (the V codes) against the E4M3 codes of the divisions, for every x;
// - int8_codes_rn (the Q and K codes) against round-half-even of the divisions, where
//   |x / delta| <= 127.
// Mismatches are counted in *count; the first one found is written to first[0..2]
// (pattern, delta index, 1).
__global__ void __launch_bounds__(256) debug_quotient_check_kernel(const float *__restrict__ deltas, int n_delta,
                                                                   int bf16, unsigned long long *count,
                                                                   unsigned int *first) {
    const int j = blockIdx.y;   // delta index
    const float delta = deltas[j];
    if (!(delta >= kQuotientMinDelta) || !(delta < 0x1p+120f)) return;
    const float y = 1.0f / delta;
    unsigned long long bad = 0;
    unsigned int bad_pat = 0;
    for (uint32_t p = blockIdx.x * blockDim.x + threadIdx.x; p < 65536u; p += gridDim.x * blockDim.x) {
        const float x = h16_to_f32(p, bf16);
        if (!isfinite(x) || fabsf(x) > 448.0f * delta) continue;
        const float2 y2 = make_float2(y, y), nd2 = make_float2(-delta, -delta);
        const float2 q = quotient2_rn(make_float2(x, -x), y2, nd2);
        const float ref = __fdiv_rn(x, delta), nref = __fdiv_rn(-x, delta);
        bool same = e4m3x4_codes_rn(x, -x, -x, x, y2, nd2) == pack_e4m3x4(ref, nref, nref, ref);
        if (fabsf(ref) >= 0x1p-20f)
            same = same && __float_as_uint(q.x) == __float_as_uint(ref) && __float_as_uint(q.y) == __float_as_uint(nref);
        if (fabsf(ref) <= 127.0f) {
            const float xs[2] = {x, -x};
            const uint32_t want = (uint32_t)(uint8_t)(int)rintf(ref) | ((uint32_t)(uint8_t)(int)rintf(nref) << 8);
            same = same && int8_codes_rn<2>(xs, y2, nd2) == want;
        }
        if (!same) {
            ++bad;
            bad_pat = p;
        }
    }
    if (bad) {
        atomicAdd(count, bad);
        if (atomicCAS(&first[2], 0u, 1u) == 0u) {
            first[0] = bad_pat;
            first[1] = (unsigned int)j;
        }
    }
}

cudaError_t launch_debug_quotient_check(const float *deltas, int n_delta, int bf16, unsigned long long *count,
                                        unsigned int *first, cudaStream_t stream) {
    debug_quotient_check_kernel<<<dim3(64, (unsigned)n_delta), 256, 0, stream>>>(deltas, n_delta, bf16, count, first);
    return cudaGetLastError();
}

cudaError_t launch_debug_quant_fp4(const float *xs, int n_rows, int d, uint8_t *codes, uint8_t *sf, float *g,
                                   cudaStream_t stream) {
    const int tiles = (n_rows + kTile - 1) / kTile;
    if (d == 128) debug_quant_fp4_kernel<128><<<tiles, 256, 0, stream>>>(xs, n_rows, codes, sf, g);
    else debug_quant_fp4_kernel<64><<<tiles, 256, 0, stream>>>(xs, n_rows, codes, sf, g);
    return cudaGetLastError();
}

template <int KIND>
__global__ void __launch_bounds__(128, 1) debug_mma_rate_kernel(int n_iter, int *status) {
    extern __shared__ uint8_t smem_raw[];
    MmaRateSmem &sm =
        *reinterpret_cast<MmaRateSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5;
    uint4 *z = reinterpret_cast<uint4 *>(sm.a);
    for (int i = threadIdx.x; i < (int)((sizeof(sm.a) + sizeof(sm.b)) / 16); i += 128) z[i] = make_uint4(0, 0, 0, 0);
    if (threadIdx.x == 0) {
        mbar_init(&sm.bar, 1);
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) { tmem_alloc(&sm.tmem_base, 256); tmem_relinquish(); }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    if (threadIdx.x == 0) {
        const uint32_t sa = smem_u32(sm.a), sb = smem_u32(sm.b);
        for (int i = 0; i < n_iter; ++i) {
            const uint32_t kk = (uint32_t)(i & 3) * 32u;
            const uint64_t ad = smem_desc(sa + kk, 1024u, 2u), bd = smem_desc(sb + kk, 1024u, 2u);
            const uint32_t acc = i > 0 ? 1u : 0u;
            if constexpr (KIND == 0) mma_e4m3_ss(tmem, ad, bd, idesc_e4m3_f32(128, 256), acc);
            else if constexpr (KIND == 1) mma_e4m3_ss(tmem, ad, bd, idesc_e4m3_f32(128, 256) & ~(3u << 4), acc);
            else if constexpr (KIND == 2) mma_s8_ss(tmem, ad, bd, idesc_s8_s32(128, 256), acc);
            else mma_f16_ss(tmem, ad, bd, idesc_f16_f32(128, 256, true), acc);
        }
        mma_commit(&sm.bar);
    }
    __syncwarp();
    mbar_wait(&sm.bar, 0, &sm.abort_flag, status, kSiteRate);
    tc_fence_after();
    __syncthreads();
    if (warp == 0) { __syncwarp(); tc_fence_after(); tmem_dealloc(tmem, 256); }
}

template <int KIND>
static cudaError_t launch_rate(int n_iter, int n_ctas, int *status, cudaStream_t stream) {
    cudaError_t e = cudaFuncSetAttribute(debug_mma_rate_kernel<KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kRateSmem);
    if (e != cudaSuccess) return e;
    debug_mma_rate_kernel<KIND><<<n_ctas, 128, kRateSmem, stream>>>(n_iter, status);
    return cudaGetLastError();
}

cudaError_t launch_debug_mma_rate(int kind, int n_iter, int n_ctas, int *status, cudaStream_t stream) {
    static_assert(sizeof(MmaRateSmem) + 1024 <= kRateSmem, "operands fit the requested shared memory");
    switch (kind) {
        case 0: return launch_rate<0>(n_iter, n_ctas, status, stream);
        case 1: return launch_rate<1>(n_iter, n_ctas, status, stream);
        case 2: return launch_rate<2>(n_iter, n_ctas, status, stream);
        default: return launch_rate<3>(n_iter, n_ctas, status, stream);
    }
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
// Diagnostic: one FP4 QK^T tile on the block-scaled tensor core (tcgen05.mma
// kind::mxf4nvf4, scale_vec::4X): S = sum over 16-channel blocks b of sfq[i][b] sfk[j][b]
// (Q4[i] . K4[j] over the block), FP32 in tensor memory.  Rows of E2M1 codes (two per
// byte, channel 2c in the low nibble) are staged K-major with the 32-byte (d = 64) or
// 64-byte (d = 128) swizzle; the E4M3 scales of each 64-channel chunk as a 512-byte atom
// (row m, block b at byte 16 (m mod 32) + 4 (m / 32) + b), copied into tensor memory by
// tcgen05.cp.  The smoothed Q / K tiles of the 4-bit mode take exactly this form
// ("SageAttention2" abstract: 4-bit QK^T; "SageAttention3: Microscaling FP4 Attention",
// listed among the notes' related papers).
// ---------------------------------------------------------------------------
template <int D>
struct Fp4Layout {
    static constexpr uint32_t row_bytes = D / 2;
    static constexpr uint32_t layout = (D == 64) ? 6u : 4u;   // UMMA 32-byte / 64-byte swizzle
    static constexpr uint32_t sbo = 8 * row_bytes;            // 8-row groups
    static constexpr int chunks = D / 64;                     // K = 64 per MMA
};
// Byte offset of 16-byte chunk c of row r in a swizzled K-major FP4 tile.
template <int D>
__device__ __forceinline__ uint32_t fp4_row_offset(uint32_t r, uint32_t c) {
    if constexpr (D == 64) return r * 32u + ((c ^ ((r >> 2) & 1u)) << 4);
    return r * 64u + ((c ^ ((r >> 1) & 3u)) << 4);
}

template <int D>
struct __align__(1024) Fp4QkSmem {
    uint8_t q[kTile * D / 2];
    uint8_t k[kTile * D / 2];
    uint8_t sfq[D / 64][512];
    uint8_t sfk[D / 64][512];
    uint64_t bar_mma;
    uint32_t tmem_base;
    int abort_flag;
};

template <int D>
__global__ void __launch_bounds__(128, 1)
    debug_qk_fp4_kernel(const uint8_t *q4, const uint8_t *k4, const uint8_t *sfq, const uint8_t *sfk, float *out,
                        int *status) {
    using L = Fp4Layout<D>;
    extern __shared__ uint8_t smem_raw[];
    Fp4QkSmem<D> &sm = *reinterpret_cast<Fp4QkSmem<D> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = threadIdx.x;
    if (threadIdx.x == 0) {
        mbar_init(&sm.bar_mma, 1);
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) { tmem_alloc(&sm.tmem_base, 256); tmem_relinquish(); }
    // row r of Q and K into the swizzled tiles; its scales into the atoms
#pragma unroll
    for (uint32_t c = 0; c < L::row_bytes / 16; ++c) {
        *reinterpret_cast<uint4 *>(sm.q + fp4_row_offset<D>(r, c)) = reinterpret_cast<const uint4 *>(q4 + (size_t)r * L::row_bytes)[c];
        *reinterpret_cast<uint4 *>(sm.k + fp4_row_offset<D>(r, c)) = reinterpret_cast<const uint4 *>(k4 + (size_t)r * L::row_bytes)[c];
    }
#pragma unroll
    for (int b = 0; b < D / 16; ++b) {
        const int at = 16 * (r & 31) + 4 * (r >> 5) + (b & 3);
        sm.sfq[b >> 2][at] = sfq[(size_t)r * (D / 16) + b];
        sm.sfk[b >> 2][at] = sfk[(size_t)r * (D / 16) + b];
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const uint32_t t_sfq = tmem + 128u, t_sfk = tmem + 144u;   // 4 columns per 64-channel chunk
    volatile int *abort_flag = &sm.abort_flag;
    if (threadIdx.x == 0) {
#pragma unroll
        for (int kc = 0; kc < L::chunks; ++kc) {
            tmem_cp_sf_atom(t_sfq + 4u * kc, sf_atom_desc(smem_u32(sm.sfq[kc])));
            tmem_cp_sf_atom(t_sfk + 4u * kc, sf_atom_desc(smem_u32(sm.sfk[kc])));
        }
        constexpr uint32_t idesc = idesc_mxf4_e4m3sf(128, 128);
#pragma unroll
        for (int kc = 0; kc < L::chunks; ++kc)
            mma_mxf4_ss(tmem, smem_desc(smem_u32(sm.q) + 32u * kc, L::sbo, L::layout),
                        smem_desc(smem_u32(sm.k) + 32u * kc, L::sbo, L::layout), idesc, t_sfq + 4u * kc,
                        t_sfk + 4u * kc, kc > 0 ? 1u : 0u);
        mma_commit(&sm.bar_mma);
    }
    __syncwarp();
    mbar_wait(&sm.bar_mma, 0, abort_flag, status, kSiteDebug);
    tc_fence_after();
    __syncthreads();
    if (*abort_flag == 0) {
#pragma unroll
        for (int c0 = 0; c0 < kTile; c0 += 32) {
            uint32_t v[32];
            tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + c0, v);
            tmem_wait_ld_regs(v);
#pragma unroll
            for (int i = 0; i < 32; ++i) out[(size_t)(warp * 32 + lane) * kTile + c0 + i] = __uint_as_float(v[i]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) { __syncwarp(); tc_fence_after(); tmem_dealloc(tmem, 256); }
}

cudaError_t launch_debug_qk_fp4(const uint8_t *q4, const uint8_t *k4, const uint8_t *sfq, const uint8_t *sfk, int d,
                                float *out, int *status, cudaStream_t stream) {
    if (d == 128) {
        const size_t smem = sizeof(Fp4QkSmem<128>) + 1024;
        cudaError_t e = cudaFuncSetAttribute(debug_qk_fp4_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        debug_qk_fp4_kernel<128><<<1, 128, smem, stream>>>(q4, k4, sfq, sfk, out, status);
    } else {
        const size_t smem = sizeof(Fp4QkSmem<64>) + 1024;
        cudaError_t e = cudaFuncSetAttribute(debug_qk_fp4_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        debug_qk_fp4_kernel<64><<<1, 128, smem, stream>>>(q4, k4, sfq, sfk, out, status);
    }
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Diagnostic: sum over tiles of P . V on the FP8 path, one FP32 accumulator
// (ACC16: an FP16 accumulator instead, the SageAttention2++ variant; the raw
// 32-bit tensor-memory words are written out).  P and V^T tiles are copied row by
// row into the 128-byte-swizzled layout the attention kernel uses for P.
// ---------------------------------------------------------------------------
template <int D>
struct __align__(1024) PvDebugSmem {
    uint8_t p[kTile * kTile];
    uint8_t v[D * kTile];
    uint64_t bar_mma;
    uint32_t tmem_base;
    int abort_flag;
};

template <int D, bool ACC16>
__global__ void __launch_bounds__(128, 1)
    debug_pv_kernel(const uint8_t *p, const uint8_t *vt, int n_tiles, float *out, int *status) {
    extern __shared__ uint8_t smem_raw[];
    PvDebugSmem<D> &sm =
        *reinterpret_cast<PvDebugSmem<D> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5;
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
            if constexpr (ACC16) {
                constexpr uint32_t idesc = idesc_e4m3_f32(128, D) & ~(3u << 4);  // D format 0: f16
#pragma unroll
                for (int kk = 0; kk < kTile / 32; ++kk)
                    mma_e4m3_ss(tmem, smem_desc(smem_u32(sm.p) + kk * 32, 1024u, 2u),
                                smem_desc(smem_u32(sm.v) + kk * 32, 1024u, 2u), idesc, (tile > 0 || kk > 0) ? 1u : 0u);
            } else {
                issue_pv<D>(tmem, smem_u32(sm.p), smem_u32(sm.v), tile > 0);
            }
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

template <int D, bool ACC16>
static cudaError_t launch_debug_pv_d(const uint8_t *p, const uint8_t *vt, int n_tiles, float *o, int *status,
                                     cudaStream_t stream) {
    const size_t smem = sizeof(PvDebugSmem<D>) + 1024;
    cudaError_t e =
        cudaFuncSetAttribute(debug_pv_kernel<D, ACC16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    debug_pv_kernel<D, ACC16><<<1, 128, smem, stream>>>(p, vt, n_tiles, o, status);
    return cudaGetLastError();
}

cudaError_t launch_debug_pv(const uint8_t *p, const uint8_t *vt, int n_tiles, int d, float *o, int *status,
                            cudaStream_t stream, int acc_f16) {
    if (d == 128)
        return acc_f16 ? launch_debug_pv_d<128, true>(p, vt, n_tiles, o, status, stream)
                       : launch_debug_pv_d<128, false>(p, vt, n_tiles, o, status, stream);
    return acc_f16 ? launch_debug_pv_d<64, true>(p, vt, n_tiles, o, status, stream)
                   : launch_debug_pv_d<64, false>(p, vt, n_tiles, o, status, stream);
}

}  // namespace sage
