// attn_fwd.cu -- fused sm_100a attention kernel of the smoothed-INT8-QK / FP8-PV
// forward (its MMA issue sequences are in attn_mma.cuh, shared with the diagnostic
// kernels of debug_kernels.cu).
//
// Method (SageAttention2, arXiv 2411.10958, abstract; SageAttention2++ verdict on
// pith.science, key_machinery): S = dQ(i) dK(j) (Q_int . K_int) + dS[t, j] on the
// INT8 tensor core; tiled online softmax ("Online normalizer calculation for
// softmax", Milakov and Gimelshein) over 128-key tiles; P~ = exp(x - m) scaled by
// Pr and rounded to E4M3; O += P8 . V8 on the FP8 tensor core, FP32 accumulation
// in tensor memory; O = acc * delta_V / (Pr l).
//
// One CTA computes two 128-row Q tiles (A = 2u, B = 2u + 1) of one head, sharing
// every K / V^T tile between them (640 threads, 20 warps):
//   warps 0-7   softmax + epilogue of tile A
//   warps 8-15  softmax + epilogue of tile B
//   warp 16     TMA producer: Q tiles once, then K tiles with their dS rows and
//               delta_K runs through one shared-memory ring
//   warp 17     tensor-memory allocation and single-thread tcgen05.mma issue
//   warp 18     TMA producer of the V^T ring
//   warp 19     idle (it completes the producer warpgroup), except in the FQ form
// Half rows: each row of a tile is held by two threads of one warp, one with its
// even and one with its odd keys (the tcgen05.ld 16x64b shape), so each scheduler
// runs four softmax warps.  Keys are stored in every 128-key tile in the order
// (even keys, odd keys) -- in P here, and in V^T and dS by the pre-pass -- so each
// thread's 64 keys are contiguous; PV is a sum over keys and does not depend on
// their order.
// Tensor memory (512 columns): S_A 0-127, S_B 128-255 (int32), O_A 256.., O_B
// 256 + d.. (fp32).  A softmax warpgroup releases its S buffer as soon as the
// scores of key tile i + 1 are in registers (it reads them while exponentiating
// tile i), so QK^T of tile i + 2 runs on the tensor core during the softmax of
// tile i + 1; the MMA issuer serves the tiles in turn with the pair (QK^T of tile
// i + 2, PV of tile i).  P is double-buffered per tile.
// In the 4-bit mode (QK4, d = 64) Q and K are E2M1 codes with E4M3 scales per 16
// channels: each QK^T is one tcgen05.mma kind::mxf4nvf4 (K = 64) whose scale atoms
// tcgen05.cp copies into tensor-memory columns 384-407, and S arrives in fp32.
// In the FQ form (opt-in: Q quantized in the kernel) warp 16 loads the caller's 16-bit
// Q tiles into the tiles' P buffers, each softmax warpgroup smooths and quantizes its
// own tile before its first scores (quantize_q_tile), and warp 19 forms the dS rows
// of every key tile from the caller's 16-bit K (ds_role).
// Every wait is bounded: a wait that runs out records SAGE_ERR_TIMEOUT in the
// status block, raises a CTA-wide abort flag that makes every role leave its loop,
// drains the copies in flight, frees tensor memory and exits.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "attn_mma.cuh"
#include "sage_device.cuh"
#include "sage_internal.h"

namespace sage {

constexpr int kAttnThreads = 640;
constexpr int kSoftmaxWarps = 16;
constexpr int kWarpK = 16, kWarpMma = 17, kWarpV = 18, kWarpDs = 19;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 256;
// 4-bit mode (d = 64): scale atoms of Q tiles A, B at 384 / 388, of K stage s at 392 + 4 s
constexpr uint32_t kTmemSfQ = 384, kTmemSfK = 392;
constexpr uint64_t kDrainNs = 50ull * 1000ull * 1000ull;
// K codes + V^T codes of the heads whose CTAs run together stay within this many
// bytes, a part of the 126 MB L2 (the rest holds the streaming Q codes, dS and O).
constexpr size_t kKvL2Budget = 48ull << 20;
// Register split (setmaxnreg): 640 threads launch with 96 registers each; the
// producer warpgroup gives back to 32 so the four softmax warpgroups can hold 112:
// 128 * 32 + 512 * 112 = 640 * 96.
constexpr uint32_t kRegsProducer = 32;
constexpr uint32_t kRegsSoftmax = 112;

// Wait-site ids recorded with a timeout.
enum { kSiteQ = 1, kSiteFull = 2, kSiteEmpty = 3, kSiteS = 4, kSiteP = 5, kSiteO = 6, kSiteSfree = 7 };

// K tiles (with their dS rows and delta_K runs) and V^T tiles travel in separate
// rings: a K slot is free once QK^T has read it and both tiles' warps have
// dequantized with its dS / delta_K, long before PV is done with the V^T tile of
// the same key tile, so the K ring can run further ahead.
// PV16 (the FP16 P / V mode): P~ and V^T are fp16, two 64-key 128-byte swizzle spans
// per row; the larger tiles leave room for one P buffer per Q tile (a tile's
// warpgroup writes P(i) once PV(i - 1) has read it) and shorter rings at d = 128.
// FQ (Q quantized in the kernel): the raw-K chunk ring of the dS warp takes the
// room of one K stage at d = 128.
template <int D, bool PV16, bool FQ = false>
struct AttnCfg {
    static constexpr int kKStages = ((PV16 || FQ) && D == 128) ? 3 : 4;
    static constexpr int kRawChunks = (D == 128 && PV16) ? 2 : 4;   // FQ: 16-key raw K chunks in flight
    static constexpr int kVStages = PV16 ? (D == 128 ? 2 : 3) : (D == 128 ? 3 : 4);
    static constexpr int kPBufs = PV16 ? 1 : 2;                     // P buffers per Q tile
    static constexpr int kPBytes = kTile * kTile * (PV16 ? 2 : 1);  // one P tile
    static constexpr int kVBytes = D * kTile * (PV16 ? 2 : 1);      // one V^T tile
};

// Shared memory of the in-kernel Q quantization and the dS warp (FQ only).
template <bool FQ, int D, int KS, int RC>
struct FqSmem {};
template <int D, int KS, int RC>
struct __align__(1024) FqSmem<true, D, KS, RC> {
    // raw K chunks: 16 keys x d of the caller's 16-bit K, as d / 64 boxes of 16 rows x
    // 128 bytes (128-byte swizzle, 2 KB each)
    uint8_t kr[RC][D / 64][16 * 128];
    // qbar of Q tiles A, B as hi / lo 16-bit numbers (rows 2x, 2x + 1), each row in
    // the order the mma.sync B operand takes it: channel 16 s + w at 16 s + 4 q + e
    // (w = 2 q + e for w < 8, w = 2 q + 8 + e - 2 for w >= 8)
    uint16_t qhl[4][D];
    float qbar[2][D];
    float wmax[2][8];
    int kr_coord[3];   // raw K coordinates: row offset, head (or head-major index), batch (-1: head-major)
    uint64_t bar_kr[RC], bar_dsfull[KS], bar_qraw, bar_qready[2];
};

template <int D, bool PV16, bool FQ = false>
struct __align__(1024) AttnSmem {
    static constexpr int KS = AttnCfg<D, PV16, FQ>::kKStages, VS = AttnCfg<D, PV16, FQ>::kVStages;
    static constexpr int RC = AttnCfg<D, PV16, FQ>::kRawChunks;
    uint8_t q[2][kTile * D];
    uint8_t k[KS][kTile * D];
    uint8_t v[VS][AttnCfg<D, PV16, FQ>::kVBytes];
    // [Q tile][key tile parity (FP8) or 0 (FP16)], keys in storage order
    uint8_t p[2][AttnCfg<D, PV16, FQ>::kPBufs][AttnCfg<D, PV16, FQ>::kPBytes];
    float ds[KS][2][kTile];          // keys in storage order
    float dk[KS][kTile / kKeyRun];
    // 4-bit mode: E4M3 scale atoms of the Q tiles and of each K stage (d = 64 only)
    alignas(128) uint8_t sfq[2][D == 64 ? 512 : 16];
    alignas(128) uint8_t sfk[KS][D == 64 ? 512 : 16];
    uint64_t bar_q, bar_kfull[KS], bar_kempty[KS], bar_vfull[VS], bar_vempty[VS];
    uint64_t bar_s[2], bar_sfree[2], bar_p[2], bar_o[2], bar_drain;
    uint32_t tmem_base;
    int abort_flag;
    int bh_kv;  // key/value head of this CTA's query head (read by the epilogue)
    FqSmem<FQ, D, KS, RC> fq;
};

// A bounded wait whose outcome is the same for all 32 lanes (so that the warp
// leaves its loop together and its .sync.aligned instructions stay converged).
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag, int *status,
                                          int site) {
    const bool ok = mbar_wait(bar, parity, abort_flag, status, site);
    return __all_sync(0xFFFFFFFFu, ok);
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

template <uint32_t N>
__device__ __forceinline__ void setmaxnreg_inc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void setmaxnreg_dec() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// Number of key tiles Q tile t sees (causal: key j visible to row i iff j <= i + off).
__device__ __forceinline__ int kv_tiles_of(int t, int Tq, int Tk, int n_q, int off, int causal) {
    if (t >= Tq) return 0;
    if (!causal) return Tk;
    const int last_key = min(t * kTile + kTile - 1, n_q - 1) + off;
    return last_key < 0 ? 0 : min(Tk, last_key / kTile + 1);
}


// ---------------------------------------------------------------------------
// Softmax + epilogue of one Q tile: 8 warps, each row held by a pair of threads
// (t, t ^ 2) of one warp, one with the row's even keys and one with its odd keys.
//
// The row's work is software-pipelined across key tiles: while the exponentials
// of tile `it` are taken (16 of the thread's keys at a time), the scores of tile
// it + 1 are read from tensor memory and dequantized, so the exponent unit and the
// ALU / FMA pipes are fed from one instruction stream.
// ---------------------------------------------------------------------------

// dS read from shared memory as inline asm, so the compiler keeps it behind the
// tensor-memory wait of its chunk instead of hoisting a whole tile's dS into
// registers.
__device__ __forceinline__ float4 lds_f32x4(const float *ptr) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(smem_u32(ptr)));
    return v;
}

// s = S * dQ dK + dS over 16 of a thread's keys (keys 2k + parity of a 32-key
// chunk), in place (S int32 -> fp32 bits); ds holds their dS contiguously (storage
// order); a_lo / a_hi scale the keys of the chunk's first / second 16-key run
// (k < 8 / k >= 8).  Returns the maximum.
// QK4: S is already fp32 (the block-scaled FP4 product), a_lo / a_hi the tile scales.
template <bool QK4>
__device__ __forceinline__ float dequant16(uint32_t (&w)[16], float a_lo, float a_hi, const float *ds) {
#pragma unroll
    for (int j = 0; j < 16; j += 4) {
        const float a = j < 8 ? a_lo : a_hi;
        const float2 a2 = make_float2(a, a);
        const float4 d4 = lds_f32x4(ds + j);
        float2 s01, s23;
        if constexpr (QK4) {
            s01 = make_float2(__uint_as_float(w[j]), __uint_as_float(w[j + 1]));
            s23 = make_float2(__uint_as_float(w[j + 2]), __uint_as_float(w[j + 3]));
        } else {
            s01 = make_float2((float)(int)w[j], (float)(int)w[j + 1]);
            s23 = make_float2((float)(int)w[j + 2], (float)(int)w[j + 3]);
        }
        const float2 y01 = __ffma2_rn(s01, a2, make_float2(d4.x, d4.y));
        const float2 y23 = __ffma2_rn(s23, a2, make_float2(d4.z, d4.w));
        w[j] = __float_as_uint(y01.x);
        w[j + 1] = __float_as_uint(y01.y);
        w[j + 2] = __float_as_uint(y23.x);
        w[j + 3] = __float_as_uint(y23.y);
    }
#define WV(j) __uint_as_float(w[j])
    const float t0 = max3f(WV(0), WV(1), WV(2)), t1 = max3f(WV(3), WV(4), WV(5)), t2 = max3f(WV(6), WV(7), WV(8));
    const float t3 = max3f(WV(9), WV(10), WV(11)), t4 = max3f(WV(12), WV(13), WV(14));
    return fmaxf(max3f(t0, t1, t2), max3f(t3, t4, WV(15)));
#undef WV
}

// p = 2^(s c + bias) (bias = log2 Pr - m c) over 16 keys: accumulates the
// unquantized p into the thread's part of the row sum and packs Pr-scaled E4M3
// codes, 4 per word.
__device__ __forceinline__ void exp16(const uint32_t (&w)[16], float2 c2, float2 b2, float2 &acc0, float2 &acc1,
                                      uint32_t (&pk)[4]) {
#pragma unroll
    for (int j = 0; j < 16; j += 4) {
        const float2 e01 = __ffma2_rn(make_float2(__uint_as_float(w[j]), __uint_as_float(w[j + 1])), c2, b2);
        const float2 e23 = __ffma2_rn(make_float2(__uint_as_float(w[j + 2]), __uint_as_float(w[j + 3])), c2, b2);
        const float2 p01 = make_float2(ex2_approx(e01.x), ex2_approx(e01.y));
        const float2 p23 = make_float2(ex2_approx(e23.x), ex2_approx(e23.y));
        acc0 = __fadd2_rn(acc0, p01);
        acc1 = __fadd2_rn(acc1, p23);
        pk[j / 4] = pack_e4m3x4(p01.x, p01.y, p23.x, p23.y);
    }
}

// The same exponentials kept as fp16 (round to nearest even, no Pr scale: bias is
// -m c), two per word, for the FP16 P / V mode.
__device__ __forceinline__ void exp16_f16(const uint32_t (&w)[16], float2 c2, float2 b2, float2 &acc0,
                                          float2 &acc1, uint32_t (&ph)[8]) {
#pragma unroll
    for (int j = 0; j < 16; j += 4) {
        const float2 e01 = __ffma2_rn(make_float2(__uint_as_float(w[j]), __uint_as_float(w[j + 1])), c2, b2);
        const float2 e23 = __ffma2_rn(make_float2(__uint_as_float(w[j + 2]), __uint_as_float(w[j + 3])), c2, b2);
        const float2 p01 = make_float2(ex2_approx(e01.x), ex2_approx(e01.y));
        const float2 p23 = make_float2(ex2_approx(e23.x), ex2_approx(e23.y));
        acc0 = __fadd2_rn(acc0, p01);
        acc1 = __fadd2_rn(acc1, p23);
        const __half2 h01 = __floats2half2_rn(p01.x, p01.y), h23 = __floats2half2_rn(p23.x, p23.y);
        ph[j / 2] = *reinterpret_cast<const uint32_t *>(&h01);
        ph[j / 2 + 1] = *reinterpret_cast<const uint32_t *>(&h23);
    }
}

// Key tile `kt` has invisible keys in this row block: the key-count tail, or the
// causal diagonal (key j visible to row i iff j <= i + off).
__device__ __forceinline__ bool tile_masked(int kt, int t, int n_kv, int off, int causal) {
    return (kt * kTile + kTile > n_kv) || (causal && kt * kTile + kTile - 1 > t * kTile + off);
}

// Sets this thread's invisible keys of key tile kt to -inf (its keys are
// 32 q + 2 k + par) and returns the maximum of its remaining scores.
__device__ __forceinline__ float mask_tile(uint32_t (&sv)[4][16], int kt, int row, int par, int n_kv, int off,
                                           int causal) {
    int lim = n_kv - 1 - kt * kTile;
    if (causal) lim = min(lim, row + off - kt * kTile);
    float mx = -INFINITY;
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            if (32 * q + 2 * k + par > lim) sv[q][k] = __float_as_uint(-INFINITY);
            mx = fmaxf(mx, __uint_as_float(sv[q][k]));
        }
    return mx;
}

// Row maximum of the two threads of a row pair.
__device__ __forceinline__ float pair_max(float v) { return fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, 2)); }

__device__ __forceinline__ uint32_t pack16x2(float lo, float hi, int out_bf16) {
    if (out_bf16) {
        __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<uint32_t *>(&h);
    }
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

// ---------------------------------------------------------------------------
// Q quantization of one Q tile inside the kernel (FQ), by the tile's 8 softmax warps
// ("SageAttention2", arXiv 2411.10958, abstract: Q smoothed per block, then quantized
// per group).  The caller's 16-bit tile sits in the tile's P buffers (TMA, 128-byte
// swizzle, d / 64 boxes of [128 rows][128 B]), which PV does not use before the
// tile's first scores exist; the codes go to the tile's Q operand.  The arithmetic
// is the pre-pass quantizer's, so the codes, delta_Q and qbar are the same bits:
//   qbar[c] = fp32(fp64 sum of the valid rows / rows)  (0 without Q smoothing),
//   x = fp32(q) - qbar (0 on rows past n_q), delta = amax_group / 127 (1 if 0),
//   code = round-half-even(x / delta).
// Also returns the row's x . kbar (the logit shift of K smoothing, for the LSE).
// Every thread of the 8 warps reaches both warpgroup barriers, whatever the outcome
// of its wait, so a failed wait cannot leave the others waiting.
// ---------------------------------------------------------------------------
template <int D, bool PV16>
__device__ __forceinline__ bool quantize_q_tile(AttnSmem<D, PV16, true> &sm, const AttnParams &p, int X, int t,
                                                int n_q, int bh, int r, int par, float &dq_out, float &shift_out,
                                                volatile int *abort_flag) {
    constexpr int kBox = kTile * 128;   // one 64-channel box of the raw tile
    const int j = threadIdx.x & 255, w8 = j >> 5, lane = j & 31;
    const int bf16 = p.out_bf16;
    const uint8_t *raw = &sm.p[X][0][0];
    const int nvalid = min(kTile, n_q - t * kTile);
    const bool ok = warp_wait(&sm.fq.bar_qraw, 0, abort_flag, p.status, kSiteQ);

    // column sums: warp w8 owns D / 8 columns, lane = column + (D / 8) * row segment
    {
        constexpr int CPW = D / 8, SEG = 32 / CPW, RPS = kTile / SEG;
        const int c = w8 * CPW + lane % CPW, seg = lane / CPW;
        const uint8_t *col = raw + (c / 64) * kBox + ((c % 64) & 7) * 2;
        const uint32_t chunk = (uint32_t)((c % 64) >> 3);
        double s0 = 0.0, s1 = 0.0;
        if (ok) {
#pragma unroll 4
            for (int i = 0; i < RPS; i += 2) {
                const int r0 = seg * RPS + i;
                const float x0 = h16_to_f32(*reinterpret_cast<const uint16_t *>(col + sw128_offset(r0, chunk)), bf16);
                const float x1 = h16_to_f32(*reinterpret_cast<const uint16_t *>(col + sw128_offset(r0 + 1, chunk)), bf16);
                s0 = __dadd_rn(s0, r0 < nvalid ? (double)x0 : 0.0);
                s1 = __dadd_rn(s1, r0 + 1 < nvalid ? (double)x1 : 0.0);
            }
        }
        double sum = __dadd_rn(s0, s1);
#pragma unroll
        for (int o = CPW; o < 32; o <<= 1) sum = __dadd_rn(sum, __shfl_xor_sync(0xFFFFFFFFu, sum, o));
        if (seg == 0) {
            const float qb = (p.use_ds && nvalid > 0) ? (float)__ddiv_rn(sum, (double)nvalid) : 0.f;
            sm.fq.qbar[X][c] = qb;
            // hi / lo 16-bit split for the dS product, in the mma.sync operand order
            const float hi = bf16 ? __bfloat162float(__float2bfloat16_rn(qb)) : __half2float(__float2half_rn(qb));
            const float lo = qb - hi;
            const uint16_t hb = bf16 ? __bfloat16_as_ushort(__float2bfloat16_rn(hi)) : __half_as_ushort(__float2half_rn(hi));
            const uint16_t lb = bf16 ? __bfloat16_as_ushort(__float2bfloat16_rn(lo)) : __half_as_ushort(__float2half_rn(lo));
            const int w = c & 15, pos = (c & ~15) + ((w & 7) >> 1) * 4 + (w >= 8 ? 2 : 0) + (w & 1);
            sm.fq.qhl[2 * X][pos] = hb;
            sm.fq.qhl[2 * X + 1][pos] = lb;
            if (ok) p.qbar_w[((size_t)bh * p.Tq + t) * D + c] = qb;
        }
    }
    named_bar_sync(1 + X, 256);

    // this thread's half row: channels [par D / 2, par D / 2 + D / 2), 8 per 16-byte chunk
    const bool valid = r < nvalid;
    const float *kbar = p.kbar + (size_t)sm.bh_kv * D + par * (D / 2);
    const float *qbar = sm.fq.qbar[X] + par * (D / 2);
    auto load8 = [&](int cc, float (&x)[8]) {   // x = Q_s of 8 channels (0 past n_q)
        const int c0 = par * (D / 2) + 8 * cc;
        const uint4 u = *reinterpret_cast<const uint4 *>(raw + (c0 / 64) * kBox + sw128_offset(r, (c0 % 64) >> 3));
        const uint32_t wv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float q = h16_to_f32((e & 1) ? (wv[e >> 1] >> 16) : (wv[e >> 1] & 0xFFFFu), bf16);
            x[e] = valid ? __fsub_rn(q, qbar[8 * cc + e]) : 0.f;
        }
    };
    float am = 0.f, shift = 0.f;
#pragma unroll
    for (int cc = 0; cc < D / 16; ++cc) {
        float x[8];
        load8(cc, x);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            am = fmaxf(am, fabsf(x[e]));
            shift = fmaf(x[e], __ldg(kbar + 8 * cc + e), shift);
        }
    }
    am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, 16));
    am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, 8));
    am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, 4));
    am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, 2));
    am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, 1));
    if (lane == 0) sm.fq.wmax[X][w8] = am;
    named_bar_sync(1 + X, 256);
    // group amax: 32 rows are the two warps of one lane quadrant, 128 rows all eight
    float gam;
    if (p.g_q == kTile) {
        gam = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) gam = fmaxf(gam, sm.fq.wmax[X][i]);
    } else {
        gam = fmaxf(sm.fq.wmax[X][w8 & 3], sm.fq.wmax[X][(w8 & 3) + 4]);
    }
    const float dl = (gam == 0.f) ? 1.f : __fdiv_rn(gam, 127.f);
    const float inv = 1.0f / dl;
    // codes: 16 channels per 16-byte chunk of the operand row (d bytes, 128- / 64-byte swizzle)
    uint8_t *qrow = sm.q[X];
    int8_t *dump = p.q8_dump ? p.q8_dump + ((size_t)bh * p.nq_pad + (size_t)t * kTile + r) * D + par * (D / 2) : nullptr;
#pragma unroll
    for (int cc = 0; cc < D / 16; cc += 2) {
        float x0[8], x1[8];
        load8(cc, x0);
        load8(cc + 1, x1);
        const float a0[4] = {x0[0], x0[1], x0[2], x0[3]}, a1[4] = {x0[4], x0[5], x0[6], x0[7]};
        const float a2[4] = {x1[0], x1[1], x1[2], x1[3]}, a3[4] = {x1[4], x1[5], x1[6], x1[7]};
        const uint4 code = make_uint4(int8_codes<4>(a0, dl, inv), int8_codes<4>(a1, dl, inv),
                                      int8_codes<4>(a2, dl, inv), int8_codes<4>(a3, dl, inv));
        const uint32_t ch = (uint32_t)((par * (D / 2) + 8 * cc) >> 4);   // 16-byte chunk of the code row
        const uint32_t off = (D == 128) ? sw128_offset((uint32_t)r, ch)
                                        : (uint32_t)r * 64u + ((ch ^ (((uint32_t)r >> 1) & 3u)) << 4);
        *reinterpret_cast<uint4 *>(qrow + off) = code;
        if (dump && ok) *reinterpret_cast<uint4 *>(dump + 8 * cc) = code;
    }
    shift += __shfl_xor_sync(0xFFFFFFFFu, shift, 2);
    if (ok && par == 0) p.dq_w[(size_t)bh * p.nq_pad + (size_t)t * kTile + r] = dl;
    dq_out = dl;
    shift_out = shift;
    // the codes are read by the tensor core: make them visible to the async proxy
    fence_proxy_async_smem();
    mbar_arrive(&sm.fq.bar_qready[X]);
    return ok;
}

// Storage position of key k of a 128-key tile: keys 32 q + 2 i + par sit at
// par * 64 + 16 q + i (the half-row order of the scores).
__device__ __forceinline__ int key_position(int k) { return (k & 1) * 64 + (k >> 5) * 16 + ((k & 31) >> 1); }

// ---------------------------------------------------------------------------
// dS warp (FQ): dS[t, j] = qbar_t . K[j] for both Q tiles and every key tile, on
// mma.sync from 16-key chunks of the caller's 16-bit K (raw-K ring, its own TMA
// loads), qbar split into hi + lo 16-bit numbers as in the pre-pass product:
// D[key][n] = sum_c K[key][c] B[c][n], B's columns (hi_A, lo_A, hi_B, lo_B, 0...),
// dS_x = D[.][2x] + D[.][2x + 1].  K enters unsmoothed: qbar_t . kbar is the same for
// every key of a row, so softmax does not see it and the LSE adds back only x . kbar.
// Results go to the dS slot of the key tile's K stage, which the stage's
// empty barrier frees; bar_dsfull[s] tells the softmax warps they are there.
// ---------------------------------------------------------------------------
template <int D, bool PV16>
__device__ __forceinline__ void ds_role(AttnSmem<D, PV16, true> &sm, const AttnParams &p, const CUtensorMap *tm_kr,
                                        int n_tiles, bool hasB, volatile int *abort_flag) {
    constexpr int KS = AttnCfg<D, PV16, true>::kKStages, RC = AttnCfg<D, PV16, true>::kRawChunks;
    constexpr int CH = kTile / 16;          // chunks per key tile
    constexpr int kChunkBytes = (D / 64) * 16 * 128;
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const bool bf16 = p.out_bf16 != 0;
    const int total = n_tiles * CH;
    // lane 0: chunk c into ring slot c % RC (coordinates from shared memory, written by
    // the kernel's set-up, so that they take no registers of this 32-register warp)
    auto issue = [&](int c) {
        const int slot = c % RC, key = (c / CH) * kTile + (c % CH) * 16 + sm.fq.kr_coord[0];
        const int hd = sm.fq.kr_coord[1], bt = sm.fq.kr_coord[2];
        mbar_arrive_expect_tx(&sm.fq.bar_kr[slot], kChunkBytes);
#pragma unroll
        for (int bx = 0; bx < D / 64; ++bx) {
            if (bt >= 0) tma_load_4d(sm.fq.kr[slot][bx], tm_kr, &sm.fq.bar_kr[slot], bx * 64, hd, key, bt);
            else tma_load_3d(sm.fq.kr[slot][bx], tm_kr, &sm.fq.bar_kr[slot], bx * 64, key, hd);
        }
    };
    if (lane == 0) {
        prefetch_tmap(tm_kr);
        for (int c = 0; c < RC && c < total; ++c) issue(c);
    }
    bool ok = warp_wait(&sm.fq.bar_qready[0], 0, abort_flag, p.status, kSiteQ);
    if (ok && hasB) ok = warp_wait(&sm.fq.bar_qready[1], 0, abort_flag, p.status, kSiteQ);
    // this lane's ldmatrix row: key (lane & 7) + 8 ((lane >> 3) & 1), 8-channel half lane >> 4
    const uint32_t lr = (uint32_t)((lane & 7) + 8 * ((lane >> 3) & 1));
    const uint32_t a_lane = smem_u32(sm.fq.kr[0][0]) + lr * 128u, a_x = lr & 7u, a_h = (uint32_t)(lane >> 4);
    const uint32_t b_lane = smem_u32(sm.fq.qhl[g < 4 ? g : 0]) + 8u * (uint32_t)q;
    int c = 0;   // chunks consumed
    for (; ok && c < total; ++c) {
        const int it = c / CH, ch = c % CH, s = it % KS, slot = c % RC;
        if (ch == 0 && it >= KS &&   // the dS slot of this key tile's K stage is free
            !warp_wait(&sm.bar_kempty[s], ((it / KS) & 1) ^ 1, abort_flag, p.status, kSiteEmpty)) {
            ok = false;
            break;
        }
        if (!warp_wait(&sm.fq.bar_kr[slot], (c / RC) & 1, abort_flag, p.status, kSiteFull)) { ok = false; break; }
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        const uint32_t a_slot = a_lane + (uint32_t)slot * kChunkBytes;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t c8 = 2u * (uint32_t)ks + a_h;   // 8-channel chunk over d
            uint32_t a0, a1, a2, a3, b0, b1;
            ldmatrix_x4(a_slot + (c8 >> 3) * 2048u + (((c8 & 7u) ^ a_x) << 4), a0, a1, a2, a3);
            asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(b0), "=r"(b1) : "r"(b_lane + 32u * ks));
            if (g >= 4) b0 = b1 = 0u;
            mma_16816(acc, a0, a1, a2, a3, b0, b1, bf16);
        }
        __syncwarp();   // every lane's reads of the slot are complete: it may be refilled
        if (lane == 0 && c + RC < total) issue(c + RC);
        if (q < 2) {    // lane q = x holds tile x's hi / lo columns for keys g, g + 8
            float *ds = sm.ds[s][q];
            ds[key_position(ch * 16 + g)] = acc[0] + acc[1];
            ds[key_position(ch * 16 + g + 8)] = acc[2] + acc[3];
        }
        if (ch == CH - 1) mbar_arrive(&sm.fq.bar_dsfull[s]);
    }
    if (!ok && lane == 0)   // let the chunk loads in flight land before the CTA exits
        for (int k = c; k < total && k < c + RC; ++k) mbar_wait_quiet(&sm.fq.bar_kr[k % RC], (k / RC) & 1, kDrainNs);
    __syncwarp();
}

template <int D, bool PV16, bool QK4, bool FQ>
__device__ __forceinline__ void softmax_role(AttnSmem<D, PV16, FQ> &sm, const AttnParams &p, uint32_t tmem, int X, int t,
                                             int n_tiles, int bh, int64_t o_base, int n_q, int n_kv, bool q_loaded,
                                             volatile int *abort_flag) {
    constexpr int KS = AttnCfg<D, PV16, FQ>::kKStages;
    const int w8 = (threadIdx.x >> 5) & 7;  // warp within the tile's eight
    const int quad = w8 & 3, half = w8 >> 2;
    const int lane = threadIdx.x & 31;
    const int par = (lane >> 1) & 1;        // this thread's key parity (tcgen05.ld 16x64b layout)
    const int r = 32 * quad + 16 * half + 8 * (lane & 1) + (lane >> 2);  // tile row = TMEM lane
    const int row = t * kTile + r;
    const uint32_t lane_base = (uint32_t)(32 * quad + 16 * half) << 16;
    const uint32_t s_tmem = tmem + lane_base + (uint32_t)X * 128u;
    const uint32_t o_tmem = tmem + lane_base + kTmemO + (uint32_t)X * D;
    const int off = n_kv - n_q;
    const int pos0 = par * (kTile / 2);  // storage position of this thread's first key of a tile
    // this thread writes output columns [par * D / 2, par * D / 2 + D / 2) of its row
    uint16_t *orow = static_cast<uint16_t *>(p.o) + o_base + (int64_t)row * p.so_n + par * (D / 2);

    // FQ: this warpgroup quantizes its own Q tile first (when the CTA loaded Q at all)
    float dq_fq = 1.f, shift_fq = 0.f;
    bool q_ok = true;
    if constexpr (FQ) {
        if (q_loaded) q_ok = quantize_q_tile<D, PV16>(sm, p, X, t, n_q, bh, r, par, dq_fq, shift_fq, abort_flag);
    }
    const bool wait_ds = FQ && p.use_ds;

    if (n_tiles == 0) {  // this tile's rows see no key: O = 0, LSE = -inf
        if (row < n_q) {
            uint4 *dst = reinterpret_cast<uint4 *>(orow);
#pragma unroll
            for (int i = 0; i < D / 16; ++i) dst[i] = make_uint4(0, 0, 0, 0);
            if (par == 0) p.lse[(size_t)bh * p.nq_pad + row] = -INFINITY;
        }
        return;
    }

    const float dq = FQ ? dq_fq : p.dq[(size_t)bh * p.nq_pad + row];
    const float c = p.scale_log2;
    const float2 c2 = make_float2(c, c);
    float m, l = 0.f, alpha = 1.f, bias;
    uint32_t sv[4][16];  // 32-key chunks of the tile, 16 of this thread's keys each

    // prologue: scores of key tile 0
    bool ok = q_ok && warp_wait(&sm.bar_s[X], 0, abort_flag, p.status, kSiteS) &&
              warp_wait(&sm.bar_kfull[0], 0, abort_flag, p.status, kSiteFull);
    if constexpr (FQ) {
        if (ok && wait_ds) ok = warp_wait(&sm.fq.bar_dsfull[0], 0, abort_flag, p.status, kSiteFull);
    }
    if (ok) {
        tc_fence_after();
        float mx[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            tmem_ld16x64b_x16(s_tmem + q * 32, sv[q]);
            tmem_wait_ld_regs16(sv[q]);
            mx[q] = dequant16<QK4>(sv[q], dq * sm.dk[0][2 * q], dq * sm.dk[0][2 * q + 1], sm.ds[0][X] + pos0 + 16 * q);
        }
        // S may take the next QK^T, and K slot 0 may be refilled: both are read now (the
        // arrival must follow the dS / delta_K reads above, since it also frees the slot)
        tc_fence_before();
        mbar_arrive(&sm.bar_sfree[X]);
        m = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
        if (tile_masked(0, t, n_kv, off, p.causal)) m = mask_tile(sv, 0, row, par, n_kv, off, p.causal);
        m = pair_max(m);
        bias = (m == -INFINITY) ? 0.f : p.log2_pr - m * c;
    }

    for (int it = 0; ok && it < n_tiles; ++it) {
        const bool has_next = it + 1 < n_tiles;
        const int sn = (it + 1) % KS;
        if (has_next) {
            if (!warp_wait(&sm.bar_s[X], (it + 1) & 1, abort_flag, p.status, kSiteS)) { ok = false; break; }
            if (!warp_wait(&sm.bar_kfull[sn], ((it + 1) / KS) & 1, abort_flag, p.status, kSiteFull)) { ok = false; break; }
            if constexpr (FQ) {
                if (wait_ds && !warp_wait(&sm.fq.bar_dsfull[sn], ((it + 1) / KS) & 1, abort_flag, p.status, kSiteFull)) {
                    ok = false;
                    break;
                }
            }
            tc_fence_after();
        }
        // exponentials of tile it, interleaved with the scores of tile it + 1 (on the
        // last tile the reads only see stale, unused values of this warp's own lanes)
        const float2 b2 = make_float2(bias, bias);
        float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
        float mx[4];
        const float *dsn = sm.ds[sn][X] + pos0;
        const float *dkn = sm.dk[sn];
        // FP8: P(it) goes to the buffer PV(it - 2) read; that PV was waited for before
        // P(it - 1).  FP16: the one buffer PV(it - 1) reads; wait for that PV first.
        uint8_t *pbuf = sm.p[X][PV16 ? 0 : (it & 1)];
        if constexpr (PV16) {
            if (it > 0 && !warp_wait(&sm.bar_o[X], (it - 1) & 1, abort_flag, p.status, kSiteO)) { ok = false; break; }
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            if constexpr (PV16) {
                // keys 16 q .. 16 q + 15 of this thread's 64-key span (its parity's half of
                // the row): two 16-byte chunks of the span's 128-byte row
                uint32_t ph[8];
                exp16_f16(sv[q], c2, b2, acc0, acc1, ph);
                uint8_t *span = pbuf + par * (kTile * 128);
                *reinterpret_cast<uint4 *>(span + sw128_offset(r, 2 * q)) = make_uint4(ph[0], ph[1], ph[2], ph[3]);
                *reinterpret_cast<uint4 *>(span + sw128_offset(r, 2 * q + 1)) = make_uint4(ph[4], ph[5], ph[6], ph[7]);
            } else {
                uint32_t pk[4];
                exp16(sv[q], c2, b2, acc0, acc1, pk);
                *reinterpret_cast<uint4 *>(pbuf + sw128_offset(r, par * 4 + q)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
            tmem_ld16x64b_x16(s_tmem + q * 32, sv[q]);
            tmem_wait_ld_regs16(sv[q]);
            mx[q] = dequant16<QK4>(sv[q], dq * dkn[2 * q], dq * dkn[2 * q + 1], dsn + 16 * q);
        }
        if (has_next) {  // tile it + 1's scores are in registers: its S buffer may take the next QK^T
            tc_fence_before();
            mbar_arrive(&sm.bar_sfree[X]);
        }
        const float2 acc = __fadd2_rn(acc0, acc1);
        l = l * alpha + (acc.x + acc.y);  // this thread's half of the row sum
        const bool rescale = (it > 0) && (alpha != 1.f);

        if (it > 0) {  // PV of the previous tile must be done before O is rescaled
            if (!warp_wait(&sm.bar_o[X], (it - 1) & 1, abort_flag, p.status, kSiteO)) { ok = false; break; }
            tc_fence_after();
        }
        if (__any_sync(0xFFFFFFFFu, rescale)) {  // this thread's half of the row's O columns
            const float2 al2 = make_float2(alpha, alpha);
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t ov[16];
                tmem_ld16x64b_x16(o_tmem + c0, ov);
                tmem_wait_ld_regs16(ov);
#pragma unroll
                for (int i = 0; i < 16; i += 2) {
                    const float2 v2 = __fmul2_rn(make_float2(__uint_as_float(ov[i]), __uint_as_float(ov[i + 1])), al2);
                    ov[i] = __float_as_uint(v2.x);
                    ov[i + 1] = __float_as_uint(v2.y);
                }
                tmem_st16x64b_x16(o_tmem + c0, ov);
            }
            tmem_wait_st();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&sm.bar_p[X]);

        if (has_next) {  // running maximum with tile it + 1
            float tmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
            if (tile_masked(it + 1, t, n_kv, off, p.causal))
                tmax = mask_tile(sv, it + 1, row, par, n_kv, off, p.causal);
            const float m_new = fmaxf(m, pair_max(tmax));
            if (m_new == -INFINITY) {
                alpha = 1.f;
                bias = 0.f;
            } else {
                alpha = ex2_approx((m - m_new) * c);
                bias = p.log2_pr - m_new * c;
            }
            m = m_new;
        }
    }
    if (ok) ok = warp_wait(&sm.bar_o[X], (n_tiles - 1) & 1, abort_flag, p.status, kSiteO);
    if (ok) {
        tc_fence_after();
        const float l_row = l + __shfl_xor_sync(0xFFFFFFFFu, l, 2);
        const float inv_l = (l_row > 0.f) ? 1.f / l_row : 0.f;
        if (par == 0 && row < n_q) {
            // l carries the factor Pr and m is in score units: the logits' log-sum-exp is
            // ln 2 (c (m + Q_s . kbar) + log2(l / Pr)), the Q_s . kbar term undoing the
            // shift that K smoothing applied to the whole row
            const size_t ri = (size_t)bh * p.nq_pad + row;
            const float shift = FQ ? shift_fq : p.qs_kbar[ri];
            p.lse[ri] = (l_row > 0.f) ? 0.6931471805599453f * (c * (m + shift) + log2f(l_row) - p.log2_pr)
                                      : -INFINITY;
        }
        const float *dv = p.dv + (size_t)sm.bh_kv * D;
        // The thread holds O columns 2v + par (v < D / 2).  Output word i of the even
        // thread is columns (2i, 2i + 1), i < D / 4; of the odd thread, columns
        // (D / 2 + 2i, D / 2 + 2i + 1): each thread swaps half its values with its pair.
#pragma unroll
        for (int cb = 0; cb < D / 64; ++cb) {
            uint32_t lo[16], hi[16];  // values v = 16 cb + k and v = D / 4 + 16 cb + k
            tmem_ld16x64b_x16(o_tmem + 32 * cb, lo);
            tmem_ld16x64b_x16(o_tmem + D / 2 + 32 * cb, hi);
            tmem_wait_ld_regs16(lo);
            tmem_wait_ld_regs16(hi);
            uint32_t out[16];  // output words for columns 32 cb + 2k (+ D / 2 on the odd thread)
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const int v_lo = 16 * cb + k, v_hi = D / 4 + 16 * cb + k;
                const float y_lo = __uint_as_float(lo[k]) * __ldg(dv + 2 * v_lo + par) * inv_l;
                const float y_hi = __uint_as_float(hi[k]) * __ldg(dv + 2 * v_hi + par) * inv_l;
                const float got = __shfl_xor_sync(0xFFFFFFFFu, par ? y_lo : y_hi, 2);
                out[k] = par ? pack16x2(got, y_hi, p.out_bf16) : pack16x2(y_lo, got, p.out_bf16);
            }
            if (row < n_q) {
                uint4 *dst = reinterpret_cast<uint4 *>(orow + 32 * cb);
#pragma unroll
                for (int i = 0; i < 4; ++i) dst[i] = make_uint4(out[4 * i], out[4 * i + 1], out[4 * i + 2], out[4 * i + 3]);
            }
        }
    }
}

// RT: sequence lengths decided at run time (a packed batch when p.cu_q is set, else
// the dense lengths); without RT the kernel serves dense batches only and reads the
// lengths straight from the parameters.  The two compile to different register
// allocations: d = 128 dense runs faster without RT, d = 64 dense with it (measured).
// FQ: Q quantized in the kernel from the caller's 16-bit Q (tm_q), dS formed in the
// kernel from the caller's 16-bit K (tm_kr) by warp 19; without FQ tm_kr is unused.
template <int D, bool RT, bool PV16, bool QK4, bool FQ>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kr,
                    const __grid_constant__ AttnParams p) {
    constexpr int KS = AttnCfg<D, PV16, FQ>::kKStages, VS = AttnCfg<D, PV16, FQ>::kVStages;
    constexpr int kPBufs = AttnCfg<D, PV16, FQ>::kPBufs, kPBytes = AttnCfg<D, PV16, FQ>::kPBytes;
    static_assert(!QK4 || (D == 64 && !PV16), "the 4-bit mode runs at d = 64 with FP8 P / V");
    static_assert(!(QK4 && FQ), "the 4-bit mode quantizes Q in the pre-pass");
    static_assert(!FQ || (size_t)kPBufs * kPBytes >= (size_t)kTile * D * 2, "a raw 16-bit Q tile fits its P buffers");
    constexpr int kQkRowBytes = QK4 ? D / 2 : D;   // bytes of one Q / K row in shared memory
    extern __shared__ uint8_t smem_raw[];
    AttnSmem<D, PV16, FQ> &sm =
        *reinterpret_cast<AttnSmem<D, PV16, FQ> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // Work item: a pair of Q tiles of one head.  The CTAs are ordered in blocks of
    // p.head_block heads and, within a block, pair-major (the pairs of rank 0 of every
    // head first; longest pairs first when causal): the CTAs in flight read the K and
    // V^T tiles of a block's heads, which stay in L2, and the long causal pairs of a
    // block start early.  The last block may hold fewer heads.
    const int n_pairs = (p.Tq + 1) / 2;
    const int blk = blockIdx.x / (n_pairs * p.head_block);
    const int r = blockIdx.x - blk * (n_pairs * p.head_block);
    const int nb = min(p.head_block, p.BH - blk * p.head_block);
    const int pair_idx = r / nb;
    const int bh = blk * p.head_block + r % nb;
    const int u = p.causal ? (n_pairs - 1 - pair_idx) : pair_idx;
    const int tA = 2 * u, tB = 2 * u + 1;
    const int b = bh / p.H, h = bh % p.H;
    const int bh_kv = b * p.H_kv + h / p.group;  // key/value head of query head h
    // Lengths of this head's sequence: a packed batch gives each sequence its own (the
    // workspace rows stay padded to the longest, p.n_q / p.n_kv)
    int n_q = p.n_q, n_kv = p.n_kv;
    int64_t o_base = (int64_t)b * p.so_b + (int64_t)h * p.so_h;
    int q_off = 0, kv_off = 0;   // first row of the sequence in a packed batch
    if (RT && p.cu_q) {
        const SeqRange sq = seq_range(p.cu_q, b, p.n_q, p.total_q), sk = seq_range(p.cu_kv, b, p.n_kv, p.total_kv);
        n_q = sq.n;
        n_kv = sk.n;
        o_base = (int64_t)sq.off * p.so_n + (int64_t)h * p.so_h;
        q_off = sq.off;
        kv_off = sk.off;
    }
    // raw-tensor coordinates (FQ): token-major maps are [batch][row][head][d] (a packed
    // batch is one batch), head-major maps [head][row][d]
    const bool tok = p.nhd || (RT && p.cu_q);
    const int b_coord = (RT && p.cu_q) ? 0 : b;
    const int Tq = (n_q + kTile - 1) / kTile, Tk = (n_kv + kTile - 1) / kTile;
    if (tA >= Tq) return;  // a pair past the end of a shorter packed sequence (the whole CTA)
    const int off = n_kv - n_q;
    const int nA = kv_tiles_of(tA, Tq, Tk, n_q, off, p.causal);
    const int nB = kv_tiles_of(tB, Tq, Tk, n_q, off, p.causal);
    const int n_tiles = max(nA, nB);
    const bool hasB = tB < Tq;

    if (threadIdx.x == 0) {
        mbar_init(&sm.bar_q, 1);
        for (int s = 0; s < KS; ++s) { mbar_init(&sm.bar_kfull[s], 1); mbar_init(&sm.bar_kempty[s], 1); }
        for (int s = 0; s < VS; ++s) { mbar_init(&sm.bar_vfull[s], 1); mbar_init(&sm.bar_vempty[s], 1); }
        for (int x = 0; x < 2; ++x) {
            mbar_init(&sm.bar_s[x], 1);
            mbar_init(&sm.bar_sfree[x], 256);  // the 8 warps of the tile
            mbar_init(&sm.bar_p[x], 256);
            mbar_init(&sm.bar_o[x], 1);
        }
        mbar_init(&sm.bar_drain, 1);
        if constexpr (FQ) {
            mbar_init(&sm.fq.bar_qraw, 1);
            mbar_init(&sm.fq.bar_qready[0], 256);
            mbar_init(&sm.fq.bar_qready[1], 256);
            for (int i = 0; i < AttnCfg<D, PV16, FQ>::kRawChunks; ++i) mbar_init(&sm.fq.bar_kr[i], 1);
            for (int i = 0; i < KS; ++i) mbar_init(&sm.fq.bar_dsfull[i], 32);
            sm.fq.kr_coord[0] = kv_off;
            sm.fq.kr_coord[1] = tok ? h / p.group : bh_kv;
            sm.fq.kr_coord[2] = tok ? b_coord : -1;
        }
        sm.abort_flag = 0;
        sm.bh_kv = bh_kv;
        fence_mbar_init();
    }
    if constexpr (FQ) {   // qbar digits of a missing tile B stay zero
        uint32_t *z = reinterpret_cast<uint32_t *>(&sm.fq.qhl[0][0]);
        for (int i = threadIdx.x; i < 4 * D / 2; i += kAttnThreads) z[i] = 0u;
    }
    if (!p.use_ds) {  // without Q smoothing the dS rows stay zero
        float *z = &sm.ds[0][0][0];
        for (int i = threadIdx.x; i < KS * 2 * kTile; i += kAttnThreads) z[i] = 0.f;
    }
    if (warp == kWarpMma && n_tiles > 0) {
        tmem_alloc(&sm.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    volatile int *abort_flag = &sm.abort_flag;

    if (warp >= kSoftmaxWarps) {
        setmaxnreg_dec<kRegsProducer>();
        if (warp == kWarpK && lane == 0 && n_tiles > 0) {
            // ---------------- TMA producer: Q tiles, then the K / dS / delta_K ring ----------------
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_k);
            if constexpr (FQ) {   // the caller's 16-bit Q tiles into the tiles' P buffers
                mbar_arrive_expect_tx(&sm.fq.bar_qraw, (hasB ? 2 : 1) * kTile * D * 2);
                for (int x = 0; x < (hasB ? 2 : 1); ++x) {
                    const int row = (x ? tB : tA) * kTile + q_off;
#pragma unroll
                    for (int bx = 0; bx < D / 64; ++bx) {
                        uint8_t *dst = &sm.p[x][0][0] + bx * (kTile * 128);
                        if (tok) tma_load_4d(dst, &tm_q, &sm.fq.bar_qraw, bx * 64, h, row, b_coord);
                        else tma_load_3d(dst, &tm_q, &sm.fq.bar_qraw, bx * 64, row, bh);
                    }
                }
            } else {
                mbar_arrive_expect_tx(&sm.bar_q, (hasB ? 2 : 1) * (kTile * kQkRowBytes + (QK4 ? 512 : 0)));
                tma_load_2d(sm.q[0], &tm_q, &sm.bar_q, 0, bh * p.nq_pad + tA * kTile);
                if (hasB) tma_load_2d(sm.q[1], &tm_q, &sm.bar_q, 0, bh * p.nq_pad + tB * kTile);
            }
            if constexpr (QK4) {
                bulk_load(sm.sfq[0], p.sfq + ((size_t)bh * p.Tq + tA) * 512, 512, &sm.bar_q);
                if (hasB) bulk_load(sm.sfq[1], p.sfq + ((size_t)bh * p.Tq + tB) * 512, 512, &sm.bar_q);
            }
            const float *ds_a = p.ds + ((size_t)bh * p.Tq + tA) * p.nk_pad;
            const float *ds_b = p.ds + ((size_t)bh * p.Tq + tB) * p.nk_pad;
            const float *dk_row = p.dk + (size_t)bh_kv * (p.nk_pad / kKeyRun);
            int issued = 0;
            for (int it = 0; it < n_tiles; ++it) {
                const int s = it % KS;
                if (it >= KS && !mbar_wait(&sm.bar_kempty[s], ((it / KS) & 1) ^ 1, abort_flag, p.status, kSiteEmpty))
                    break;
                issued = it + 1;
                if (p.fault_inject && it == 0) continue;  // diagnostic: leave slot 0 unsignalled
                const bool dsA = !FQ && p.use_ds && it < nA, dsB = !FQ && p.use_ds && it < nB;
                const uint32_t bytes = kTile * kQkRowBytes + (dsA ? kTile * 4 : 0) + (dsB ? kTile * 4 : 0) +
                                       (kTile / kKeyRun) * 4 + (QK4 ? 512 : 0);
                mbar_arrive_expect_tx(&sm.bar_kfull[s], bytes);
                tma_load_2d(sm.k[s], &tm_k, &sm.bar_kfull[s], 0, bh_kv * p.nk_pad + it * kTile);
                if constexpr (QK4) bulk_load(sm.sfk[s], p.sfk + ((size_t)bh_kv * p.Tk + it) * 512, 512, &sm.bar_kfull[s]);
                if (dsA) bulk_load(sm.ds[s][0], ds_a + it * kTile, kTile * 4, &sm.bar_kfull[s]);
                if (dsB) bulk_load(sm.ds[s][1], ds_b + it * kTile, kTile * 4, &sm.bar_kfull[s]);
                bulk_load(sm.dk[s], dk_row + it * (kTile / kKeyRun), (kTile / kKeyRun) * 4, &sm.bar_kfull[s]);
            }
            if (*abort_flag) {  // let the copies in flight land before the CTA exits
                if constexpr (FQ) mbar_wait_quiet(&sm.fq.bar_qraw, 0, kDrainNs);
                else mbar_wait_quiet(&sm.bar_q, 0, kDrainNs);
                for (int it = max(0, issued - KS); it < issued; ++it) {
                    if (p.fault_inject && it == 0) continue;
                    mbar_wait_quiet(&sm.bar_kfull[it % KS], (it / KS) & 1, kDrainNs);
                }
            }
        } else if (warp == kWarpV && lane == 0 && n_tiles > 0) {
            // ---------------- TMA producer: the V^T ring ----------------
            prefetch_tmap(&tm_v);
            int issued = 0;
            for (int it = 0; it < n_tiles; ++it) {
                const int s = it % VS;
                if (it >= VS && !mbar_wait(&sm.bar_vempty[s], ((it / VS) & 1) ^ 1, abort_flag, p.status, kSiteEmpty))
                    break;
                issued = it + 1;
                mbar_arrive_expect_tx(&sm.bar_vfull[s], AttnCfg<D, PV16>::kVBytes);
                if constexpr (PV16) {  // two 64-key spans of fp16
                    tma_load_2d(sm.v[s], &tm_v, &sm.bar_vfull[s], it * kTile, bh_kv * D);
                    tma_load_2d(sm.v[s] + D * 128, &tm_v, &sm.bar_vfull[s], it * kTile + 64, bh_kv * D);
                } else {
                    tma_load_2d(sm.v[s], &tm_v, &sm.bar_vfull[s], it * kTile, bh_kv * D);
                }
            }
            if (*abort_flag)
                for (int it = max(0, issued - VS); it < issued; ++it)
                    mbar_wait_quiet(&sm.bar_vfull[it % VS], (it / VS) & 1, kDrainNs);
        } else if (warp == kWarpMma && lane == 0 && n_tiles > 0) {
            // ------------------------------ MMA issuer ------------------------------
            // Q tile x at q_s + x * kTile * D; P buffer (x, b) at p_s + (x * kPBufs + b) * kPBytes
            const uint32_t q_s = smem_u32(sm.q[0]), p_s = smem_u32(sm.p[0][0]);
            // QK^T of Q tile x against K stage ks (the 4-bit mode: one block-scaled MMA whose
            // scale atoms were copied to tensor memory beforehand)
            auto qk = [&](int x, int ks) {
                if constexpr (QK4) {
                    mma_mxf4_ss(tmem + (uint32_t)x * 128u, smem_desc(q_s + (uint32_t)x * (kTile * D), 256u, 6u),
                                smem_desc(smem_u32(sm.k[ks]), 256u, 6u), idesc_mxf4_e4m3sf(128, 128),
                                tmem + kTmemSfQ + 4u * x, tmem + kTmemSfK + 4u * ks, 0u);
                } else {
                    issue_qk<D>(tmem + (uint32_t)x * 128u, q_s + (uint32_t)x * (kTile * D), smem_u32(sm.k[ks]));
                }
            };
            // 4-bit mode: the scale atom of K stage ks into tensor memory (before its QK^T)
            auto sf_k = [&](int ks) {
                if constexpr (QK4) tmem_cp_sf_atom(tmem + kTmemSfK + 4u * ks, sf_atom_desc(smem_u32(sm.sfk[ks])));
            };
            bool ok = FQ || mbar_wait(&sm.bar_q, 0, abort_flag, p.status, kSiteQ);
            if (ok) ok = mbar_wait(&sm.bar_kfull[0], 0, abort_flag, p.status, kSiteFull);
            if (ok) {
                tc_fence_after();
                if constexpr (QK4) {
                    for (int x = 0; x < 2; ++x)
                        if ((x ? nB : nA) > 0) tmem_cp_sf_atom(tmem + kTmemSfQ + 4u * x, sf_atom_desc(smem_u32(sm.sfq[x])));
                }
                sf_k(0);
                for (int x = 0; ok && x < 2; ++x)
                    if ((x ? nB : nA) > 0) {
                        if constexpr (FQ) {   // the warpgroup has written this tile's codes
                            ok = mbar_wait(&sm.fq.bar_qready[x], 0, abort_flag, p.status, kSiteQ);
                            if (!ok) break;
                            tc_fence_after();
                        }
                        qk(x, 0);
                        mma_commit(&sm.bar_s[x]);
                    }
            }
            // QK^T of key tile 1 as soon as a warpgroup holds tile 0's scores; K slot 0
            // is released once both warpgroups have dequantized tile 0
            if (ok && n_tiles > 1) ok = mbar_wait(&sm.bar_kfull[1 % KS], (1 / KS) & 1, abort_flag, p.status, kSiteFull);
            if (ok && n_tiles > 1) {
                tc_fence_after();
                sf_k(1 % KS);
            }
            for (int x = 0; ok && x < 2; ++x) {
                const int nx = x ? nB : nA;
                if (nx <= 0) continue;
                ok = mbar_wait(&sm.bar_sfree[x], 0, abort_flag, p.status, kSiteSfree);
                if (ok && nx > 1) {
                    tc_fence_after();
                    qk(x, 1 % KS);
                    mma_commit(&sm.bar_s[x]);
                }
            }
            if (ok) mma_commit(&sm.bar_kempty[0]);
            // Steady state, per key tile it and Q tile x: QK^T of tile it + 2 once x's
            // warpgroup holds tile it + 1's scores, then PV of tile it once its P is in
            // shared memory (a warpgroup releases the two close together).
            for (int it = 0; ok && it < n_tiles; ++it) {
                const int k1 = (it + 1) % KS, k2 = (it + 2) % KS, sv = it % VS;
                if (it + 2 < n_tiles) {
                    if (!mbar_wait(&sm.bar_kfull[k2], ((it + 2) / KS) & 1, abort_flag, p.status, kSiteFull)) break;
                    tc_fence_after();
                    sf_k(k2);
                }
                bool brk = false, v_ready = false;
                for (int x = 0; x < 2; ++x) {
                    const int nx = x ? nB : nA;
                    if (it + 1 < nx) {
                        if (!mbar_wait(&sm.bar_sfree[x], (it + 1) & 1, abort_flag, p.status, kSiteSfree)) { brk = true; break; }
                        if (it + 2 < nx) {
                            tc_fence_after();
                            qk(x, k2);
                            mma_commit(&sm.bar_s[x]);
                        }
                    }
                    if (it < nx) {
                        if (!v_ready) {
                            if (!mbar_wait(&sm.bar_vfull[sv], (it / VS) & 1, abort_flag, p.status, kSiteFull)) { brk = true; break; }
                            v_ready = true;
                        }
                        if (!mbar_wait(&sm.bar_p[x], it & 1, abort_flag, p.status, kSiteP)) { brk = true; break; }
                        tc_fence_after();
                        const uint32_t pb = p_s + (uint32_t)(x * kPBufs + (PV16 ? 0 : (it & 1))) * kPBytes;
                        if constexpr (PV16) issue_pv16<D>(tmem + kTmemO + (uint32_t)x * D, pb, smem_u32(sm.v[sv]), it > 0);
                        else issue_pv<D>(tmem + kTmemO + (uint32_t)x * D, pb, smem_u32(sm.v[sv]), it > 0);
                        mma_commit(&sm.bar_o[x]);
                    }
                }
                if (brk) break;
                if (it + 1 < n_tiles) mma_commit(&sm.bar_kempty[k1]);  // tile it + 1 dequantized by both warpgroups
                mma_commit(&sm.bar_vempty[sv]);                         // once PV(it) has read V^T(it)
            }
            mma_commit(&sm.bar_drain);
            mbar_wait_quiet(&sm.bar_drain, 0, kDrainNs);
        } else if (FQ && warp == kWarpDs && n_tiles > 0 && p.use_ds) {
            // ------------------------------ dS warp ------------------------------
            if constexpr (FQ)
                ds_role<D, PV16>(sm, p, &tm_kr, n_tiles, hasB, abort_flag);
        }
        // all roles meet here before tensor memory is released
        tc_fence_before();
        __syncthreads();
        if (warp == kWarpMma && n_tiles > 0) {
            __syncwarp();
            tc_fence_after();
            tmem_dealloc(tmem, kTmemCols);
        }
        return;
    }
    setmaxnreg_inc<kRegsSoftmax>();
    // one copy of the softmax code serves both tiles (instruction-cache footprint)
    const int X = warp >> 3;
    if (X == 0 || hasB)
        softmax_role<D, PV16, QK4, FQ>(sm, p, tmem, X, X ? tB : tA, X ? nB : nA, bh, o_base, n_q, n_kv, n_tiles > 0,
                                       abort_flag);
    tc_fence_before();
    __syncthreads();
}

template <int D, bool RT, bool PV16, bool QK4 = false, bool FQ = false>
static cudaError_t launch_attention_d(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                      const CUtensorMap &tkr, const AttnParams &p, cudaStream_t stream) {
    const size_t smem = sizeof(AttnSmem<D, PV16, FQ>) + 1024;
    static_assert(sizeof(AttnSmem<D, PV16, FQ>) + 1024 <= 227 * 1024, "shared memory of one CTA");
    cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<D, RT, PV16, QK4, FQ>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((p.Tq + 1) / 2) * (unsigned)p.BH;
    // Heads per block of the CTA order: as many key/value heads as fit kKvL2Budget
    // bytes of K codes + V^T codes (+ the caller's 16-bit K that the dS warp reads),
    // times the query heads that share each.
    AttnParams pp = p;
    const size_t kv_head_bytes =
        (size_t)p.nk_pad * D * ((PV16 ? 2 : 1) + (QK4 ? 0.5 : 1.0) + ((FQ && p.use_ds) ? 2.0 : 0.0));
    const size_t kv_heads = kv_head_bytes ? kKvL2Budget / kv_head_bytes : 0;
    const size_t hb = (kv_heads < 1 ? 1 : kv_heads) * (size_t)p.group;
    pp.head_block = (int)(hb < (size_t)p.BH ? hb : (size_t)p.BH);
    if (pp.head_block < 1) pp.head_block = 1;
    attn_fwd_kernel<D, RT, PV16, QK4, FQ><<<grid, kAttnThreads, smem, stream>>>(tq, tk, tv, tkr, pp);
    return cudaGetLastError();
}

cudaError_t launch_attention(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                             const CUtensorMap &tkr, const AttnParams &p, int d, cudaStream_t stream) {
    if (p.fp4) {   // the 4-bit mode: d = 64, FP8 P / V (checked by the callers)
        if (d != 64 || p.pv16 || p.fused_q) return cudaErrorInvalidValue;
        return launch_attention_d<64, true, false, true>(tq, tk, tv, tkr, p, stream);
    }
    if (p.fused_q) {   // Q quantized in the kernel
        if (p.pv16) {
            if (d == 128) return launch_attention_d<128, true, true, false, true>(tq, tk, tv, tkr, p, stream);
            return launch_attention_d<64, true, true, false, true>(tq, tk, tv, tkr, p, stream);
        }
        if (d == 128) {
            if (p.cu_q) return launch_attention_d<128, true, false, false, true>(tq, tk, tv, tkr, p, stream);
            return launch_attention_d<128, false, false, false, true>(tq, tk, tv, tkr, p, stream);
        }
        return launch_attention_d<64, true, false, false, true>(tq, tk, tv, tkr, p, stream);
    }
    if (p.pv16) {
        if (d == 128) return launch_attention_d<128, true, true>(tq, tk, tv, tkr, p, stream);
        return launch_attention_d<64, true, true>(tq, tk, tv, tkr, p, stream);
    }
    if (d == 128) {
        if (p.cu_q) return launch_attention_d<128, true, false>(tq, tk, tv, tkr, p, stream);
        return launch_attention_d<128, false, false>(tq, tk, tv, tkr, p, stream);
    }
    return launch_attention_d<64, true, false>(tq, tk, tv, tkr, p, stream);
}

}  // namespace sage
