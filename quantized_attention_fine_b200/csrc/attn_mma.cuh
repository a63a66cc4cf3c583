// attn_mma.cuh -- the tcgen05.mma issue sequences of the attention kernel (QK^T on
// the INT8 tensor core, PV on the FP8 tensor core), shared with the diagnostic
// kernels that check them ("SageAttention2", arXiv 2411.10958, abstract: INT8 QK^T,
// FP8 P V).
#pragma once

#include "sage_device.cuh"
#include "sage_internal.h"

namespace sage {

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

// O[d_tmem] (+)= P_tile . V_tile in the FP16 P / V mode: P is 128 rows x 128 keys
// of fp16 and V^T d rows x 128 keys of fp16, each stored as two 64-key spans of
// 128-byte rows (128-byte swizzle; span 1 follows span 0); 8 tcgen05.mma kind::f16
// (f16 x f16, FP32 accumulator) with M = 128, N = d, K = 16.
template <int D>
__device__ __forceinline__ void issue_pv16(uint32_t d_tmem, uint32_t p_saddr, uint32_t v_saddr, bool accumulate) {
    constexpr uint32_t idesc = idesc_f16_f32(128, D, false);
#pragma unroll
    for (int span = 0; span < 2; ++span)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            const uint64_t a = smem_desc(p_saddr + span * (kTile * 128) + kk * 32, 1024u, 2u);
            const uint64_t b = smem_desc(v_saddr + span * (D * 128) + kk * 32, 1024u, 2u);
            mma_f16_ss(d_tmem, a, b, idesc, (accumulate || span > 0 || kk > 0) ? 1u : 0u);
        }
}

}  // namespace sage
