// sage_device.cuh -- sm_100a device building blocks written as inline PTX:
// mbarriers with bounded waits, TMA (tensor and bulk) loads, tensor-memory
// allocation / load / store, tcgen05.mma issue, shared-memory matrix descriptors,
// and the INT8 quantizer shared by the pre-pass and the attention prologue.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sage {

// Error codes written to the workspace status block (same values as sage.h).
constexpr int kErrTimeout = 5;
// Bounded waits give up after this many nanoseconds of %globaltimer.
constexpr uint64_t kWaitLimitNs = 1000ull * 1000ull * 1000ull;

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Record the first device-side error of a launch: status[0] = code, status[1] = site.
__device__ __forceinline__ void record_error(int *status, int code, int site) {
    if (status != nullptr && atomicCAS(status, 0, code) == 0) atomicExch(status + 1, site);
}

// Wait until the phase with `parity` of `bar` has completed.  Gives up (returns
// false) when the CTA-wide abort flag is raised or after kWaitLimitNs, in which
// case it records SAGE_ERR_TIMEOUT with `site` and raises the abort flag.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                          int *status, int site) {
    const uint32_t a = smem_u32(bar);
    if (mbar_test(a, parity)) return true;
    const uint64_t t0 = globaltimer();
    for (uint32_t it = 1;; ++it) {
        if (mbar_test(a, parity)) return true;
        if ((it & 31) == 0) {
            if (*abort_flag) return false;
            if (globaltimer() - t0 > kWaitLimitNs) {
                record_error(status, kErrTimeout, site);
                *abort_flag = 1;
                return false;
            }
        }
    }
}

// Same, without recording anything: used to drain in-flight copies on the abort path.
__device__ __forceinline__ void mbar_wait_quiet(uint64_t *bar, uint32_t parity, uint64_t limit_ns) {
    const uint32_t a = smem_u32(bar);
    const uint64_t t0 = globaltimer();
    while (!mbar_test(a, parity)) {
        if (globaltimer() - t0 > limit_ns) return;
    }
}

// ---------------------------------------------------------------------------
// TMA
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(void *smem_dst, const CUtensorMap *map, uint64_t *bar, int x,
                                            int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
        ::"r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}
__device__ __forceinline__ void tma_load_3d(void *smem_dst, const CUtensorMap *map, uint64_t *bar, int x, int y,
                                            int z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];"
        ::"r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
        : "memory");
}
__device__ __forceinline__ void tma_load_4d(void *smem_dst, const CUtensorMap *map, uint64_t *bar, int x, int y,
                                            int z, int w) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], [%2];"
        ::"r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z),
          "r"(w)
        : "memory");
}
// Contiguous global -> shared copy; dst, src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(void *smem_dst, const void *gsrc, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_u32(smem_dst)), "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
// Tiled TMA store shared -> global (bulk-group completion), and its group control.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap *map, const void *smem_src, int x, int y, int z) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];"
                 ::"l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(smem_src)), "r"(x), "r"(y), "r"(z)
                 : "memory");
}
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, const void *smem_src, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];"
                 ::"l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(smem_src)), "r"(x), "r"(y)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until at most N committed store groups still read shared memory / are still pending.
template <int N>
__device__ __forceinline__ void bulk_wait_group_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
template <int N>
__device__ __forceinline__ void bulk_wait_group() {
    asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}
// Barrier over `count` threads (a multiple of 32) on hardware barrier `id` (1..15).
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
// Make generic-proxy shared-memory writes visible to the async proxy (tensor core).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Tensor memory
// ---------------------------------------------------------------------------
// Warp-wide.  Writes the allocated base address to *dst (shared memory).
__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 lanes x 32 bit, 32 consecutive columns: thread i of the warp receives lane
// (lane base of taddr + i), columns [col, col + 32) of taddr.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
          "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
// tcgen05.ld writes its destination registers asynchronously; they may be read
// only after tcgen05.wait::ld.  Tying the registers to the wait keeps the compiler
// from hoisting any use above it.
#define SAGE_R32(r)                                                                                     \
    "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),     \
        "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),        \
        "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),      \
        "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),      \
        "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
__device__ __forceinline__ void tmem_wait_ld_regs(uint32_t (&r)[32]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;" : SAGE_R32(r)::"memory");
}
// The same for 16 registers.
__device__ __forceinline__ void tmem_wait_ld_regs16(uint32_t (&r)[16]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                   "+r"(r[15])::"memory");
}

// 16 lanes x 64 bit shape, 16 repetitions: thread t of the warp receives lane
// (lane base of taddr + 8 (t & 1) + (t >> 2)) and, for k = 0..15, column
// (col + 2k + ((t >> 1) & 1)): the two threads t and t ^ 2 share a lane, one holding
// its even and the other its odd columns.
__device__ __forceinline__ void tmem_ld16x64b_x16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x64b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_st16x64b_x16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.16x64b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
          "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05.mma
// ---------------------------------------------------------------------------
// Instruction descriptor fields: [4,6) D format, [7,10) A format, [10,13) B format,
// [15] A major (0 = K), [16] B major, [17,23) N >> 3, [24,29) M >> 4.
__host__ __device__ constexpr uint32_t idesc_s8_s32(int M, int N) {
    return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N) {
    return (1u << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// kind::f16 with 16-bit A and B of the same type (bf16 when `bf16`, else f16), f32 D.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N, bool bf16) {
    return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

// Shared-memory matrix descriptor of a K-major operand tile whose rows are one
// swizzle span wide (128 B with layout 2 = 128-byte swizzle, 64 B with layout 4 =
// 64-byte swizzle), rows packed densely so 8-row groups are `sbo` bytes apart.
// Fields: [0,14) addr >> 4, [16,30) LBO >> 4 (unused here), [32,46) SBO >> 4,
// [46,48) version 1, [49,52) base offset 0, [61,64) layout.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t sbo, uint32_t layout) {
    uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1u << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)layout << 61;
    return d;
}

__device__ __forceinline__ void mma_s8_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void mma_e4m3_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void mma_f16_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Block-scaled FP4 (kind::mxf4nvf4): E2M1 A and B (K-major, two codes per byte), one
// unsigned E4M3 scale per 16 elements of K (scale_vec::4X, K = 64 per instruction), FP32
// D.  Fields as above, plus [4,6) B scale-factor id and [29,31) A scale-factor id (the
// byte offset of the scales inside their tensor-memory word: 0 here), [23] scale format
// (0 = E4M3), [31] K size (0 = 64); A and B format 1 = E2M1.
__host__ __device__ constexpr uint32_t idesc_mxf4_e4m3sf(int M, int N) {
    return (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ void mma_mxf4_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}
// Shared-memory descriptor of a 512-byte scale-factor atom: 32 rows of 16 bytes, no
// swizzle, 8-row core matrices 128 bytes apart (the K-major interleaved layout).
__device__ __forceinline__ uint64_t sf_atom_desc(uint32_t saddr) {
    uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1u << 16;
    d |= (uint64_t)(128u >> 4) << 32;
    d |= (uint64_t)1u << 46;
    return d;
}
// Copy a scale-factor atom (32 rows of 16 bytes) into 4 tensor-memory columns at
// `taddr`, every lane quadrant receiving the same 32 rows: lane 32 q + l holds atom row
// l.  Row m's four scales are then found in lane m, column taddr + m / 32, which is
// where kind::mxf4nvf4 with scale_vec::4X reads them.
__device__ __forceinline__ void tmem_cp_sf_atom(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// Arrive once on `bar` when all previously issued tcgen05.mma of this thread complete.
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// ---------------------------------------------------------------------------
// Number formats
// ---------------------------------------------------------------------------
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// Four fp32 -> four E4M3 bytes (byte i = value i), round to nearest even, saturating.
__device__ __forceinline__ uint32_t pack_e4m3x4(float a0, float a1, float a2, float a3) {
    uint32_t r;
    asm("{\n\t.reg .b16 lo, hi;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 lo, %2, %1;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;\n\t"
        "mov.b32 %0, {lo, hi};\n\t}"
        : "=r"(r)
        : "f"(a0), "f"(a1), "f"(a2), "f"(a3));
    return r;
}

// Value of an E4M3 code (exact, via the hardware E4M3 -> f16 conversion).
__device__ __forceinline__ float e4m3_value(uint8_t code) {
    uint32_t h2;
    asm("{\n\t.reg .b16 c;\n\tcvt.u16.u32 c, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, c;\n\t}" : "=r"(h2) : "r"((uint32_t)code));
    return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}
// Two E2M1 codes (round to nearest even, saturating): `lo` in bits 0-3, `hi` in 4-7.
__device__ __forceinline__ uint32_t e2m1x2(float hi, float lo) {
    uint32_t r;
    asm("{\n\t.reg .b8 b;\n\tcvt.rn.satfinite.e2m1x2.f32 b, %1, %2;\n\tcvt.u32.u8 %0, b;\n\t}" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// One 16-bit element (bf16 when `bf16`, else fp16) as fp32, exactly.
__device__ __forceinline__ float h16_to_f32(uint32_t bits, int bf16) {
    return bf16 ? __uint_as_float(bits << 16) : __half2float(__ushort_as_half((unsigned short)bits));
}

// Correctly rounded fp32 quotients x / delta of a pair of values, without a division
// per value, by Markstein's theorem (P. Markstein, "Computation of elementary
// functions on the IBM RISC System/6000 processor", IBM J. Res. Develop. 34, 1990):
// with y = RN(1 / delta) and q = RN(x y), which lies within an ulp of x / delta, the
// remainder x - q delta is exact in one fma, and RN(q + (x - q delta) y) = RN(x / delta)
// as long as nothing underflows.  Callers take this path only when delta >=
// kQuotientMinDelta = 2^-60.  Then a quotient of at least 2^-20 has |x| >= 2^-80, so
// that it and the remainder (about 2^-24 |x|) are normal numbers and the theorem
// applies; a smaller quotient rounds to the code 0 (INT8 or E4M3) whether exact or as
// computed here.  (x comes from the group whose amax sets delta, so x y cannot
// overflow.)
constexpr float kQuotientMinDelta = 0x1p-60f;
__device__ __forceinline__ float2 quotient2_rn(float2 x, float2 y, float2 neg_delta) {
    const float2 q = __fmul2_rn(x, y);
    const float2 r = __ffma2_rn(q, neg_delta, x);
    return __ffma2_rn(r, y, q);
}

// x's magnitude with s's sign bit.
__device__ __forceinline__ float with_sign_of(float x, float s) {
    return __uint_as_float((__float_as_uint(x) & 0x7FFFFFFFu) | (__float_as_uint(s) & 0x80000000u));
}

// Four E4M3 codes (byte i = value i; round to nearest even, saturating) of the
// correctly rounded quotients x_i / delta for delta >= kQuotientMinDelta; y =
// RN(1 / delta).  A quotient takes its dividend's sign: that changes nothing but the
// quotient of -0, which the correction step turns into +0 (+0 + -0 rounds to +0),
// while -0 / delta is -0, whose code is 0x80.
__device__ __forceinline__ uint32_t e4m3x4_codes_rn(float x0, float x1, float x2, float x3, float2 y,
                                                    float2 neg_delta) {
    const float2 a = quotient2_rn(make_float2(x0, x1), y, neg_delta);
    const float2 b = quotient2_rn(make_float2(x2, x3), y, neg_delta);
    return pack_e4m3x4(with_sign_of(a.x, x0), with_sign_of(a.y, x1), with_sign_of(b.x, x2), with_sign_of(b.y, x3));
}

// INT8 codes (packed little-endian) of round-half-even(RN(x_v / delta)) for delta >=
// kQuotientMinDelta: the quotients by quotient2_rn, rounded on the FMA pipe (RN(t +
// 1.5 * 2^23) holds round-half-even(t) in its low mantissa byte, as a two's-complement
// code).  y = RN(1 / delta); delta = amax / 127 keeps |t| below 127.5.
template <int VEC>
__device__ __forceinline__ uint32_t int8_codes_rn(const float (&xs)[VEC], float2 y, float2 neg_delta) {
    constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
    const float2 mg = make_float2(kMagic, kMagic);
    uint32_t m[4] = {0, 0, 0, 0};
#pragma unroll
    for (int v = 0; v < VEC; v += 2) {
        const float2 t = __fadd2_rn(quotient2_rn(make_float2(xs[v], xs[v + 1]), y, neg_delta), mg);
        m[v] = __float_as_uint(t.x);
        m[v + 1] = __float_as_uint(t.y);
    }
    const uint32_t lo = __byte_perm(m[0], m[1], 0x0040);
    if constexpr (VEC == 4) return __byte_perm(lo, __byte_perm(m[2], m[3], 0x0040), 0x5410);
    return lo & 0xFFFFu;
}

// INT8 codes of four values by IEEE division (round-half-even of x / delta), packed
// little-endian: the near-tie path of int8_codes, kept out of line so that the common
// path carries none of the division code.
static __device__ __noinline__ uint32_t int8_codes4_div(float x0, float x1, float x2, float x3, float delta) {
    constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
    const uint32_t m0 = __float_as_uint(__fdiv_rn(x0, delta) + kMagic);
    const uint32_t m1 = __float_as_uint(__fdiv_rn(x1, delta) + kMagic);
    const uint32_t m2 = __float_as_uint(__fdiv_rn(x2, delta) + kMagic);
    const uint32_t m3 = __float_as_uint(__fdiv_rn(x3, delta) + kMagic);
    return __byte_perm(__byte_perm(m0, m1, 0x0040), __byte_perm(m2, m3, 0x0040), 0x5410);
}

// INT8 codes of VEC values, round-half-even of the IEEE fp32 quotient xs / delta,
// packed little-endian.
// - For |xs / delta| <= 128, t = RN(xs * RN(1 / delta)) lies within 2.3e-5 of the
//   correctly rounded quotient, so when t is at least 2^-15 (3.05e-5) away from a
//   half-integer both round to the same integer; only the rare near-tie takes the
//   IEEE division.
// - Rounding is done on the FMA pipe: m = RN(t + 1.5 * 2^23) holds round-half-even(t)
//   in its low mantissa bits, so its low byte is the two's-complement code, and
//   m - 1.5 * 2^23 is that integer exactly (so t - it is exact too).
// - delta = amax / 127 bounds |t| by 127 (1 + 3 * 2^-24) < 127.5, so the codes never
//   leave [-127, 127] and the clamp of the definition never binds.
// Pairs of values go through the packed fp32x2 operations (each lane rounds as the
// scalar operation does).
template <int VEC>
__device__ __forceinline__ uint32_t int8_codes(const float (&xs)[VEC], float delta, float inv_delta) {
    static_assert(VEC == 2 || VEC == 4, "two or four values");
    constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
    const float2 inv2 = make_float2(inv_delta, inv_delta);
    const float2 mg = make_float2(kMagic, kMagic), nmg = make_float2(-kMagic, -kMagic);
    const float2 neg1 = make_float2(-1.f, -1.f);
    uint32_t m[4] = {0, 0, 0, 0};
    float dev = 0.f;   // largest |t - round(t)|
#pragma unroll
    for (int v = 0; v < VEC; v += 2) {
        const float2 t = __fmul2_rn(make_float2(xs[v], xs[v + 1]), inv2);
        const float2 tm = __fadd2_rn(t, mg);
        const float2 e = __ffma2_rn(__fadd2_rn(tm, nmg), neg1, t);
        dev = fmaxf(dev, fmaxf(fabsf(e.x), fabsf(e.y)));
        m[v] = __float_as_uint(tm.x);
        m[v + 1] = __float_as_uint(tm.y);
    }
    if (dev > 0.5f - 0x1p-15f) {
        if constexpr (VEC == 4) return int8_codes4_div(xs[0], xs[1], xs[2], xs[3], delta);
        return int8_codes4_div(xs[0], xs[1], 0.f, 0.f, delta) & 0xFFFFu;
    }
    const uint32_t lo = __byte_perm(m[0], m[1], 0x0040);
    if constexpr (VEC == 4) return __byte_perm(lo, __byte_perm(m[2], m[3], 0x0040), 0x5410);
    return lo & 0xFFFFu;
}

// ---------------------------------------------------------------------------
// Warp-level matrix multiply (mma.sync) for small side products
// ---------------------------------------------------------------------------
// Four 8 x 8 matrices of 16-bit elements from shared memory: lane l gives the row
// address of row l % 8 of matrix l / 8; register i of every lane receives its part of
// matrix i (lane t: row t / 4, elements 2 (t % 4), 2 (t % 4) + 1).
__device__ __forceinline__ void ldmatrix_x4(uint32_t saddr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(saddr)
                 : "memory");
}
// D (16 x 8, fp32) += A (16 x 16, row-major) . B (16 x 8, column-major), 16-bit A and B
// of the same type (bf16 when `bf16`, else fp16).  Lane t = 4 g + q holds
// a = {A[g][2q..], A[g + 8][2q..], A[g][2q + 8..], A[g + 8][2q + 8..]},
// b = {B[2q..][g], B[2q + 8..][g]}, d = {D[g][2q], D[g][2q + 1], D[g + 8][2q], D[g + 8][2q + 1]}.
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1, bool bf16) {
    if (bf16)
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
            "{%0, %1, %2, %3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    else
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
            "{%0, %1, %2, %3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 128-byte swizzle of a tile with 128-byte rows: byte offset of 16-byte chunk `c`
// of row `r` (the pattern TMA writes with CU_TENSOR_MAP_SWIZZLE_128B and the
// tensor core reads with layout 2).  The tile must start on a 1024-byte boundary.
__device__ __forceinline__ uint32_t sw128_offset(uint32_t r, uint32_t c) {
    return r * 128u + (((c ^ (r & 7u)) & 7u) << 4);
}

}  // namespace sage
