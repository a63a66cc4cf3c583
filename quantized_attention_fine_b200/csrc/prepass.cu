// prepass.cu -- smoothing and quantization pre-pass of the SageAttention2-style
// forward ("SageAttention2", arXiv 2411.10958, abstract: smoothing of Q and K,
// fine-grained Q/K quantization, FP8 V; per-channel V scale from the
// pith.science verdict on arXiv 2505.21136, key_machinery).
//
// Bandwidth-bound kernels (the dS product is in ds_gemm.cu); the three quantization
// kernels stream their input through TMA rings (see below):
//   kv_stats     per (key/value head, 512-token chunk): fp64 partial sums of K per
//                channel and per-channel max |V|.
//   kv_finalize  per key/value head: kbar = fp32(sum / n_kv); delta_V = max|V| / Vr.
//   quant_q      per (head, 128-row block): qbar (fp64 mean of the valid rows,
//                rounded to fp32), Q_s = Q - qbar in fp32, group amax, INT8 codes, and
//                per row Q_s . kbar (the logit shift of K smoothing, for the row LSE).
//   quant_k      per (head, 128-key tile): K_s = K - kbar, INT8 codes per group,
//                delta_K per 16-key run.
//   quant_v      per (head, 128-key tile): V / delta_V -> E4M3, written transposed
//                ([channel][position], keys in the tile storage order: even, then odd);
//                in the FP16 P / V mode V -> fp16 (round to nearest even), same layout.
// Every code decision (INT8 rounding, E4M3 rounding) is made on the IEEE fp32
// quotient x / delta, rounded to nearest even, so that it is reproducible on the
// host.  The quotient is formed without a division per element (quotient2_rn, by
// Markstein's correction of x * RN(1 / delta)), and by IEEE division for groups whose
// scale is below 2^-60.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "sage_device.cuh"
#include "sage_internal.h"

namespace sage {

namespace {

// VEC consecutive 16-bit elements (bf16 when BF16, else fp16) as fp32, exactly.
template <int VEC, bool BF16>
__device__ __forceinline__ void load_row_slice(const uint16_t *p, float (&x)[VEC]) {
    uint32_t u[VEC / 2];
    if constexpr (VEC == 4) {
        const uint2 w = *reinterpret_cast<const uint2 *>(p);
        u[0] = w.x;
        u[1] = w.y;
    } else {
        u[0] = *reinterpret_cast<const uint32_t *>(p);
    }
#pragma unroll
    for (int j = 0; j < VEC / 2; ++j) {
        if constexpr (BF16) {
            x[2 * j] = __uint_as_float(u[j] << 16);
            x[2 * j + 1] = __uint_as_float(u[j] & 0xFFFF0000u);
        } else {
            const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&u[j]));
            x[2 * j] = f.x;
            x[2 * j + 1] = f.y;
        }
    }
}

// The same with the type chosen at run time (bf16 when `bf16`, else fp16).
template <int VEC>
__device__ __forceinline__ void load_row_slice_rt(const uint16_t *p, int bf16, float (&x)[VEC]) {
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

// Sums each of 16 per-lane values over the warp's 32 lanes (a reduce-scatter: every
// exchange halves the values a lane still holds, 16 shuffles in all).  Returns, in
// lane l, the total of value l >> 1.
__device__ __forceinline__ float warp_sum16_scatter(float (&v)[16]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int w = 8; w >= 1; w >>= 1) {  // exchange with the lane 2 w away: keep half
        const bool up = (lane & (2 * w)) != 0;
#pragma unroll
        for (int k = 0; k < w; ++k) {
            const float send = up ? v[k] : v[k + w];
            const float keep = up ? v[k + w] : v[k];
            v[k] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, 2 * w);
        }
    }
    return v[0] + __shfl_xor_sync(0xFFFFFFFFu, v[0], 1);
}

template <int VEC>
__device__ __forceinline__ void store_codes(int8_t *dst, uint32_t packed) {
    if constexpr (VEC == 4) *reinterpret_cast<uint32_t *>(dst) = packed;
    else *reinterpret_cast<uint16_t *>(dst) = (uint16_t)packed;
}

}  // namespace

// Quantization kernels: persistent CTAs of 8 warps stream 128-row tiles (one
// head's rows or keys) through a ring of shared-memory stages filled by TMA, so the
// loads of the next tiles are in flight while a tile is reduced and quantized.
// Warp w owns rows 16w .. 16w + 15 of a tile; lane l owns channels l*VEC ...
constexpr int kQuantThreads = 256;
constexpr int kQuantWarps = kQuantThreads / 32;
constexpr int kRowsPerWarp = kTile / kQuantWarps;   // 16 = one delta_K run
constexpr int kSitePrepass = 31;
constexpr uint64_t kPrepassDrainNs = 50ull * 1000ull * 1000ull;

template <int D>
struct QuantRing {
    static constexpr int kStages = (D == 128) ? 3 : 4;
    static constexpr uint32_t kTileBytes = kTile * D * 2;
    static constexpr size_t kSmemBytes = kStages * kTileBytes + 128;
};

// TMA load of work unit u (row tile t = u % T of head bh = u / T) of a 16-bit
// [BH][n][d] (head-major) or [B][n][H][d] (token-major) tensor; rows past n read 0.
// A packed batch (cu not null) is token-major [1][total][H][d]: tile t of sequence b
// starts at token cu[b] + 128 t (its rows past the sequence belong to the next one and
// are masked by the consumer).
__device__ __forceinline__ void load_rows_tile(const CUtensorMap *tm, int nhd, int H, int T, int u, void *dst,
                                               uint64_t *bar, uint32_t bytes, const int *cu, int n_max, int total) {
    const int bh = u / T, t = u % T;
    mbar_arrive_expect_tx(bar, bytes);
    if (cu) tma_load_4d(dst, tm, bar, 0, bh % H, seq_range(cu, bh / H, n_max, total).off + t * kTile, 0);
    else if (nhd) tma_load_4d(dst, tm, bar, 0, bh % H, t * kTile, bh / H);
    else tma_load_3d(dst, tm, bar, 0, t * kTile, bh);
}

// Ring bookkeeping shared by the three kernels: thread 0 primes kStages loads; the
// k-th unit of this CTA sits in stage k % kStages.
template <int D>
struct RingCtl {
    uint16_t *ring;
    uint64_t *full;
    int n_units, T, H, nhd;
    const CUtensorMap *tm;
    const int *cu;   // packed batch offsets, or null
    int n_max, total;
    __device__ __forceinline__ uint16_t *stage(int k) const { return ring + (size_t)(k % QuantRing<D>::kStages) * kTile * D; }
    __device__ __forceinline__ void issue(int k) const {  // load this CTA's k-th unit, if any
        const int u = blockIdx.x + k * gridDim.x;
        if (u < n_units)
            load_rows_tile(tm, nhd, H, T, u, stage(k), &full[k % QuantRing<D>::kStages], QuantRing<D>::kTileBytes,
                           cu, n_max, total);
    }
    __device__ __forceinline__ bool wait(int k, volatile int *abort_flag, int *status) const {
        return __all_sync(0xFFFFFFFFu, mbar_wait(&full[k % QuantRing<D>::kStages], (k / QuantRing<D>::kStages) & 1,
                                                  abort_flag, status, kSitePrepass));
    }
    // on the abort path: let the loads still in flight land before the CTA exits
    __device__ __forceinline__ void drain(int k_next) const {
        for (int k = k_next; k < k_next + QuantRing<D>::kStages; ++k)
            if ((int)(blockIdx.x + k * gridDim.x) < n_units)
                mbar_wait_quiet(&full[k % QuantRing<D>::kStages], (k / QuantRing<D>::kStages) & 1, kPrepassDrainNs);
    }
};

// ring_base: where the ring starts (128-byte aligned); null = the start of dynamic
// shared memory, rounded up.
template <int D>
__device__ __forceinline__ RingCtl<D> ring_setup(const CUtensorMap *tm, int nhd, int H, int T, int BH, uint64_t *full,
                                                 volatile int *abort_flag, const int *cu, int n_max, int total,
                                                 uint8_t *ring_base = nullptr) {
    extern __shared__ uint8_t smem_raw[];
    RingCtl<D> rc;
    rc.ring = ring_base ? reinterpret_cast<uint16_t *>(ring_base)
                        : reinterpret_cast<uint16_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    rc.full = full;
    rc.n_units = BH * T;
    rc.T = T;
    rc.H = H;
    rc.nhd = nhd;
    rc.tm = tm;
    rc.cu = cu;
    rc.n_max = n_max;
    rc.total = total;
    if (threadIdx.x == 0) {
        for (int s = 0; s < QuantRing<D>::kStages; ++s) mbar_init(&full[s], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        prefetch_tmap(tm);
        for (int k = 0; k < QuantRing<D>::kStages; ++k) rc.issue(k);
    }
    return rc;
}

// FP4 (block-scaled E2M1) codes of this warp's 16 rows of a 128-row tile with tile
// scale g (the microscaling form of the 4-bit Q / K of "SageAttention2", abstract;
// "SageAttention3: Microscaling FP4 Attention" among the notes' related papers): per
// row and 16 channels the E4M3 scale sf = E4M3(fp32(fp32(amax / g) / 6)) (1.0 for an
// all-zero block, 2^-9 where it rounds to zero), per element the E2M1 code of the IEEE
// quotient x / fp32(g sf).  Codes go to codes_tile ([128][D/2], channel 2c in the low
// nibble of byte c); the scales into the tile's 512-byte atoms (row m, block b at byte
// 16 (m mod 32) + 4 (m / 32) + (b mod 4) of atom b / 4), the layout tcgen05.cp moves into
// tensor memory for kind::mxf4nvf4.
template <int D>
__device__ __forceinline__ void fp4_rows(const float (&x)[kRowsPerWarp][D / 32], float g, uint8_t *codes_tile,
                                         uint8_t *atoms_tile, int warp, int lane) {
    constexpr int VEC = D / 32, LPB = 16 / VEC;   // lanes per 16-channel block
#pragma unroll
    for (int i = 0; i < kRowsPerWarp; ++i) {
        const int r = warp * kRowsPerWarp + i;
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
        if (lane % LPB == 0) {
            const int b = lane / LPB;
            atoms_tile[(b >> 2) * 512 + 16 * (r & 31) + 4 * (r >> 5) + (b & 3)] = sc;
        }
        uint32_t packed = 0;   // VEC codes, 4 bits each, channel lane * VEC + v at bits 4 v
#pragma unroll
        for (int v = 0; v < VEC; v += 2)
            packed |= e2m1x2(__fdiv_rn(x[i][v + 1], delta), __fdiv_rn(x[i][v], delta)) << (4 * v);
        uint8_t *dst = codes_tile + (size_t)r * (D / 2) + lane * (VEC / 2);
        if constexpr (VEC == 4) *reinterpret_cast<uint16_t *>(dst) = (uint16_t)packed;
        else *dst = (uint8_t)packed;
    }
}

// Largest |x| over the 16-row groups of warps [w0, w0 + n) of this tile.
__device__ __forceinline__ float group_amax(const float *wmax, int w0, int n) {
    float am = 0.f;
    for (int w = w0; w < w0 + n; ++w) am = fmaxf(am, wmax[w]);
    return am;
}

// ---------------------------------------------------------------------------
template <int D, bool BF16>
__global__ void __launch_bounds__(256) kv_stats_kernel(const PrepassArgs a) {
    constexpr int VEC = D / 32;
    __shared__ double s_sum[8][D];
    __shared__ float s_max[8][D];
    // one-dimensional grid (head-major), so any head count fits: block = bh * n_chunks + chunk
    const int chunk = (int)(blockIdx.x % (unsigned)a.shape.n_chunks), bh = (int)(blockIdx.x / (unsigned)a.shape.n_chunks);
    const int b = bh / a.shape.H_kv, h = bh % a.shape.H_kv;  // key/value head
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const SeqRange sr = seq_range(a.cu_kv, b, a.shape.n_kv, a.shape.total_kv);
    const int64_t base = a.cu_kv ? (int64_t)sr.off * a.skv.n + h * a.skv.h : b * a.skv.b + h * a.skv.h;
    const int j0 = chunk * kStatChunk;
    const int j1 = min(j0 + kStatChunk, sr.n);
    double ks[VEC];
    float vm[VEC];
#pragma unroll
    for (int v = 0; v < VEC; ++v) { ks[v] = 0.0; vm[v] = 0.f; }
    const uint16_t *kp = a.k ? static_cast<const uint16_t *>(a.k) + base + lane * VEC : nullptr;
    const uint16_t *vp = a.v ? static_cast<const uint16_t *>(a.v) + base + lane * VEC : nullptr;
    constexpr int U = 4;   // rows whose loads are issued before the first is used
    int j = j0 + warp;
    for (; j + 8 * (U - 1) < j1; j += 8 * U) {
        float xk[U][VEC], xv[U][VEC];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (kp) load_row_slice<VEC, BF16>(kp + (int64_t)(j + 8 * u) * a.skv.n, xk[u]);
            if (vp) load_row_slice<VEC, BF16>(vp + (int64_t)(j + 8 * u) * a.skv.n, xv[u]);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (kp) {
#pragma unroll
                for (int v = 0; v < VEC; ++v) ks[v] = __dadd_rn(ks[v], (double)xk[u][v]);
            }
            if (vp) {
#pragma unroll
                for (int v = 0; v < VEC; ++v) vm[v] = fmaxf(vm[v], fabsf(xv[u][v]));
            }
        }
    }
    for (; j < j1; j += 8) {
        float x[VEC];
        if (kp) {
            load_row_slice<VEC, BF16>(kp + (int64_t)j * a.skv.n, x);
#pragma unroll
            for (int v = 0; v < VEC; ++v) ks[v] = __dadd_rn(ks[v], (double)x[v]);
        }
        if (vp) {
            load_row_slice<VEC, BF16>(vp + (int64_t)j * a.skv.n, x);
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
    const int n_kv = seq_range(a.cu_kv, bh / a.shape.H_kv, a.shape.n_kv, a.shape.total_kv).n;
    if (a.k) {
        const double *part = reinterpret_cast<const double *>(a.ws + a.L.ksum_part) + (size_t)bh * nc * D + c;
        double s = 0.0;
        for (int ch = 0; ch < nc; ++ch) s = __dadd_rn(s, part[(size_t)ch * D]);
        const float kb = (a.smooth_k && n_kv > 0) ? (float)__ddiv_rn(s, (double)n_kv) : 0.f;
        reinterpret_cast<float *>(a.ws + a.L.kbar)[(size_t)bh * D + c] = kb;
    }
    if (a.v) {
        const float *part = reinterpret_cast<const float *>(a.ws + a.L.vmax_part) + (size_t)bh * nc * D + c;
        float m = 0.f;
        for (int ch = 0; ch < nc; ++ch) m = fmaxf(m, part[(size_t)ch * D]);
        reinterpret_cast<float *>(a.ws + a.L.dv)[(size_t)bh * D + c] =
            (m == 0.f || a.pv16) ? 1.f : __fdiv_rn(m, a.v_range);  // FP16 V carries no scale
    }
}

// ---------------------------------------------------------------------------
// FP4: the 4-bit mode (a separate instantiation, so that the INT8 kernel carries
// none of its code).
template <int D, bool FP4, bool BF16>
__global__ void __launch_bounds__(kQuantThreads, 2) quant_q_kernel(const __grid_constant__ PrepassArgs a) {
    constexpr int VEC = D / 32, RPW = kRowsPerWarp;
    __shared__ uint64_t s_full[QuantRing<D>::kStages];
    __shared__ double s_sum[kQuantWarps][D];
    __shared__ float s_qbar[D];
    __shared__ float s_wmax[kQuantWarps];
    __shared__ int s_abort;
    const Shape &S = a.shape;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int *status = reinterpret_cast<int *>(a.ws + a.L.status);
    const RingCtl<D> rc = ring_setup<D>(&a.tm_q, a.nhd, S.H, S.Tq, S.BH, s_full, &s_abort, a.cu_q, S.n_q, S.total_q);
    int k = 0;
    for (;; ++k) {
        const int u = blockIdx.x + k * gridDim.x;
        if (u >= rc.n_units) break;
        const int bh = u / S.Tq, t = u % S.Tq;
        // kbar of this query head's key/value head (0 without K, i.e. no keys), loaded
        // before the tile is waited for
        float kb[VEC];
        {
            const int bh_kv = (bh / S.H) * S.H_kv + (bh % S.H) / (S.H / S.H_kv);
            const float *kbar = reinterpret_cast<const float *>(a.ws + a.L.kbar) + (size_t)bh_kv * D + lane * VEC;
#pragma unroll
            for (int v = 0; v < VEC; ++v) kb[v] = a.k ? kbar[v] : 0.f;
        }
        const int r0 = t * kTile, nvalid = min(kTile, seq_range(a.cu_q, bh / S.H, S.n_q, S.total_q).n - r0);
        if (!rc.wait(k, &s_abort, status)) break;
        if (nvalid <= 0) {  // a tile past the end of a shorter packed sequence: nothing to do
            __syncthreads();
            if (threadIdx.x == 0) rc.issue(k + QuantRing<D>::kStages);
            continue;
        }
        const uint16_t *tile = rc.stage(k) + lane * VEC;
        float x[RPW][VEC];
        double ps[VEC];
#pragma unroll
        for (int v = 0; v < VEC; ++v) ps[v] = 0.0;
#pragma unroll
        for (int i = 0; i < RPW; ++i) {
            const int r = warp * RPW + i;
            load_row_slice<VEC, BF16>(tile + r * D, x[i]);
            if (r < nvalid) {
#pragma unroll
                for (int v = 0; v < VEC; ++v) ps[v] = __dadd_rn(ps[v], (double)x[i][v]);
            }
        }
#pragma unroll
        for (int v = 0; v < VEC; ++v) s_sum[warp][lane * VEC + v] = ps[v];
        __syncthreads();  // the stage is in registers: refill it
        if (threadIdx.x == 0) rc.issue(k + QuantRing<D>::kStages);
        if (threadIdx.x < D) {  // qbar: fp64 mean of the valid rows, rounded to fp32
            const int c = threadIdx.x;
            double sum = 0.0;
#pragma unroll
            for (int w = 0; w < kQuantWarps; ++w) sum = __dadd_rn(sum, s_sum[w][c]);
            // a full tile divides by 128, which the product with 2^-7 does exactly
            const double mean = (nvalid == kTile) ? sum * (1.0 / kTile) : __ddiv_rn(sum, (double)nvalid);
            const float qb = a.smooth_q ? (float)mean : 0.f;
            s_qbar[c] = qb;
            reinterpret_cast<float *>(a.ws + a.L.qbar)[((size_t)bh * S.Tq + t) * D + c] = qb;
        }
        __syncthreads();
        float2 nqb[VEC / 2];   // -qbar of this lane's channels: x + (-qbar) is x - qbar exactly
#pragma unroll
        for (int v = 0; v < VEC; v += 2) nqb[v / 2] = make_float2(-s_qbar[lane * VEC + v], -s_qbar[lane * VEC + v + 1]);
        float am = 0.f;
#pragma unroll
        for (int i = 0; i < RPW; ++i) {
#pragma unroll
            for (int v = 0; v < VEC; v += 2) {
                const float2 xs = __fadd2_rn(make_float2(x[i][v], x[i][v + 1]), nqb[v / 2]);
                x[i][v] = xs.x;
                x[i][v + 1] = xs.y;
            }
            if (warp * RPW + i >= nvalid) {   // rows past the sequence (warp-uniform)
#pragma unroll
                for (int v = 0; v < VEC; ++v) x[i][v] = 0.f;
            }
#pragma unroll
            for (int v = 0; v < VEC; ++v) am = fmaxf(am, fabsf(x[i][v]));
        }
        // this lane's part of Q_s . kbar for each of the warp's rows, channel by channel
        // (rows taken in pairs by the packed fma)
        float shift[RPW];
#pragma unroll
        for (int i = 0; i < RPW; i += 2) {
            float2 sh = make_float2(0.f, 0.f);
#pragma unroll
            for (int v = 0; v < VEC; ++v) sh = __ffma2_rn(make_float2(x[i][v], x[i + 1][v]), make_float2(kb[v], kb[v]), sh);
            shift[i] = sh.x;
            shift[i + 1] = sh.y;
        }
        static_assert(RPW == 16, "one shift value per row of the warp's 16");
        const float row_shift = warp_sum16_scatter(shift);  // row warp * RPW + (lane >> 1)
        if ((lane & 1) == 0)
            reinterpret_cast<float *>(a.ws + a.L.qs_kbar)[(size_t)bh * S.nq_pad + r0 + warp * RPW + (lane >> 1)] = row_shift;
        am = warp_max(am);
        if (lane == 0) s_wmax[warp] = am;
        __syncthreads();
        const int gw = a.g_q / RPW;  // warps per quantization group (g_q = 32 or 128)
        const float gam = group_amax(s_wmax, (warp / gw) * gw, gw);
        if constexpr (FP4) {   // 4-bit Q: the tile scale takes delta_Q's place
            const float g = (gam == 0.f) ? 1.f : __fdiv_rn(gam, 2688.f);
            if (lane < RPW) reinterpret_cast<float *>(a.ws + a.L.dq)[(size_t)bh * S.nq_pad + r0 + warp * RPW + lane] = g;
            fp4_rows<D>(x, g, a.ws + a.L.q8 + ((size_t)bh * S.nq_pad + r0) * (D / 2),
                        a.ws + a.L.sfq + ((size_t)bh * S.Tq + t) * (D / 64) * 512, warp, lane);
            continue;
        }
        const float dl = (gam == 0.f) ? 1.f : __fdiv_rn(gam, 127.f);
        if (lane < RPW) reinterpret_cast<float *>(a.ws + a.L.dq)[(size_t)bh * S.nq_pad + r0 + warp * RPW + lane] = dl;
        int8_t *q8 = reinterpret_cast<int8_t *>(a.ws + a.L.q8) + ((size_t)bh * S.nq_pad + r0 + warp * RPW) * D + lane * VEC;
        if (dl >= kQuotientMinDelta) {
            const float y = 1.0f / dl;
            const float2 y2 = make_float2(y, y), nd2 = make_float2(-dl, -dl);
#pragma unroll
            for (int i = 0; i < RPW; ++i) store_codes<VEC>(q8 + (size_t)i * D, int8_codes_rn<VEC>(x[i], y2, nd2));
        } else {   // a group of tiny values: IEEE divisions
#pragma unroll
            for (int i = 0; i < RPW; ++i)
                store_codes<VEC>(q8 + (size_t)i * D, int8_codes4_div(x[i][0], x[i][1], VEC == 4 ? x[i][VEC - 2] : 0.f,
                                                                     VEC == 4 ? x[i][VEC - 1] : 0.f, dl));
        }
    }
    if (s_abort && threadIdx.x == 0) rc.drain(k);
}

// ---------------------------------------------------------------------------
template <int D, bool FP4, bool BF16>
__global__ void __launch_bounds__(kQuantThreads, 2) quant_k_kernel(const __grid_constant__ PrepassArgs a) {
    constexpr int VEC = D / 32, RPW = kRowsPerWarp;
    __shared__ uint64_t s_full[QuantRing<D>::kStages];
    __shared__ float s_wmax[2][kQuantWarps];
    __shared__ int s_abort;
    const Shape &S = a.shape;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int *status = reinterpret_cast<int *>(a.ws + a.L.status);
    const RingCtl<D> rc =
        ring_setup<D>(&a.tm_k, a.nhd, S.H_kv, S.Tk, S.BH_kv, s_full, &s_abort, a.cu_kv, S.n_kv, S.total_kv);
    int k = 0;
    for (;; ++k) {
        const int u = blockIdx.x + k * gridDim.x;
        if (u >= rc.n_units) break;
        const int bh = u / S.Tk, jt = u % S.Tk;
        // minus this unit's K mean (x + (-kbar) is x - kbar exactly), loaded before the
        // tile is waited for
        float2 nkb[VEC / 2];
        {
            const float *kbar = reinterpret_cast<const float *>(a.ws + a.L.kbar) + (size_t)bh * D + lane * VEC;
#pragma unroll
            for (int v = 0; v < VEC; v += 2) nkb[v / 2] = make_float2(-kbar[v], -kbar[v + 1]);
        }
        const int j0 = jt * kTile, nvalid = min(kTile, seq_range(a.cu_kv, bh / S.H_kv, S.n_kv, S.total_kv).n - j0);
        if (!rc.wait(k, &s_abort, status)) break;
        if (nvalid <= 0) {  // a tile past the end of a shorter packed sequence
            __syncthreads();
            if (threadIdx.x == 0) rc.issue(k + QuantRing<D>::kStages);
            continue;
        }
        const uint16_t *tile = rc.stage(k) + lane * VEC;
        float x[RPW][VEC];
        float am = 0.f;
#pragma unroll
        for (int i = 0; i < RPW; ++i) {
            const int r = warp * RPW + i;
            load_row_slice<VEC, BF16>(tile + r * D, x[i]);
#pragma unroll
            for (int v = 0; v < VEC; v += 2) {
                const float2 xs = __fadd2_rn(make_float2(x[i][v], x[i][v + 1]), nkb[v / 2]);
                x[i][v] = xs.x;
                x[i][v + 1] = xs.y;
            }
            if (r >= nvalid) {   // keys past the sequence (warp-uniform)
#pragma unroll
                for (int v = 0; v < VEC; ++v) x[i][v] = 0.f;
            }
#pragma unroll
            for (int v = 0; v < VEC; ++v) am = fmaxf(am, fabsf(x[i][v]));
        }
        am = warp_max(am);
        if (lane == 0) s_wmax[k & 1][warp] = am;
        __syncthreads();  // the stage is in registers: refill it
        if (threadIdx.x == 0) rc.issue(k + QuantRing<D>::kStages);
        const int gw = a.g_k / RPW;  // warps per quantization group (g_k = 16 or 128)
        const float gam = group_amax(s_wmax[k & 1], (warp / gw) * gw, gw);
        if constexpr (FP4) {   // 4-bit K: the tile scale takes delta_K's place in every 16-key run
            const float g = (gam == 0.f) ? 1.f : __fdiv_rn(gam, 2688.f);
            if (lane == 0)
                reinterpret_cast<float *>(a.ws + a.L.dk)[(size_t)bh * (S.nk_pad / kKeyRun) + (j0 + warp * RPW) / kKeyRun] = g;
            fp4_rows<D>(x, g, a.ws + a.L.k8 + ((size_t)bh * S.nk_pad + j0) * (D / 2),
                        a.ws + a.L.sfk + ((size_t)bh * S.Tk + jt) * (D / 64) * 512, warp, lane);
            continue;
        }
        const float dl = (gam == 0.f) ? 1.f : __fdiv_rn(gam, 127.f);
        if (lane == 0)  // one delta_K per 16-key run = this warp's rows
            reinterpret_cast<float *>(a.ws + a.L.dk)[(size_t)bh * (S.nk_pad / kKeyRun) + (j0 + warp * RPW) / kKeyRun] = dl;
        int8_t *k8 = reinterpret_cast<int8_t *>(a.ws + a.L.k8) + ((size_t)bh * S.nk_pad + j0 + warp * RPW) * D + lane * VEC;
        if (dl >= kQuotientMinDelta) {
            const float y = 1.0f / dl;
            const float2 y2 = make_float2(y, y), nd2 = make_float2(-dl, -dl);
#pragma unroll
            for (int i = 0; i < RPW; ++i) store_codes<VEC>(k8 + (size_t)i * D, int8_codes_rn<VEC>(x[i], y2, nd2));
        } else {   // a group of tiny values: IEEE divisions
#pragma unroll
            for (int i = 0; i < RPW; ++i)
                store_codes<VEC>(k8 + (size_t)i * D, int8_codes4_div(x[i][0], x[i][1], VEC == 4 ? x[i][VEC - 2] : 0.f,
                                                                     VEC == 4 ? x[i][VEC - 1] : 0.f, dl));
        }
    }
    if (s_abort && threadIdx.x == 0) rc.drain(k);
}

// V codes of a 128-key tile, written transposed ([channel][position]) in the tile's
// storage order: key j of a tile sits at position (j & 1) * 64 + (j >> 1) (even keys
// first, then odd keys), the order in which the attention kernel's threads hold P.
// Lane l holds the 16 keys of its warp for channels l*VEC ..; their 8 even and 8 odd
// codes per channel are two 8-byte pieces of that channel's row of V^T.
// The E4M3 V^T tile is built in shared memory ([d channels][128 positions], the
// 128-byte swizzle TMA uses) and written with one tensor store, rather than as 8-byte
// pieces scattered over d rows of the workspace.
// Dynamic shared memory (the kernel has no static part, so it starts on the shared
// window's own boundary): the V^T tile, the ring, the ring's barriers and abort flag.
// Should the start not fall on a 1024-byte boundary (the swizzle's period), the tile
// is written with plain stores instead (same bytes).
template <int D>
struct QuantVSmem {
    static constexpr size_t kStageBytes = (size_t)D * kTile;
    static constexpr size_t kRingBytes = (size_t)QuantRing<D>::kStages * QuantRing<D>::kTileBytes;
    static constexpr size_t kBytes = kStageBytes + kRingBytes + 8 * QuantRing<D>::kStages + 16;
};

template <int D>
__global__ void __launch_bounds__(kQuantThreads, 2) quant_v_kernel(const __grid_constant__ PrepassArgs a) {
    constexpr int VEC = D / 32, RPW = kRowsPerWarp;
    static_assert(RPW == 16, "a lane stores 16 keys of a channel as one 16-byte piece");
    const Shape &S = a.shape;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int *status = reinterpret_cast<int *>(a.ws + a.L.status);
    extern __shared__ uint8_t smem_raw[];   // (no alignment claimed: checked below)
    uint8_t *vts = smem_raw;
    uint64_t *s_full = reinterpret_cast<uint64_t *>(smem_raw + QuantVSmem<D>::kStageBytes + QuantVSmem<D>::kRingBytes);
    int *s_abort = reinterpret_cast<int *>(s_full + QuantRing<D>::kStages);
    const RingCtl<D> rc = ring_setup<D>(&a.tm_v, a.nhd, S.H_kv, S.Tk, S.BH_kv, s_full, s_abort, a.cu_kv, S.n_kv,
                                        S.total_kv, smem_raw + QuantVSmem<D>::kStageBytes);
    const bool staged = !a.pv16 && (smem_u32(smem_raw) & 1023u) == 0;
    if (threadIdx.x == 0 && staged) prefetch_tmap(&a.tm_vt);
    int k = 0;
    for (;; ++k) {
        const int u = blockIdx.x + k * gridDim.x;
        if (u >= rc.n_units) break;
        const int bh = u / S.Tk, jt = u % S.Tk;
        // this unit's per-channel scales, loaded before the tile is waited for
        float dv[VEC];
#pragma unroll
        for (int v = 0; v < VEC; ++v)
            dv[v] = a.pv16 ? 1.f : reinterpret_cast<const float *>(a.ws + a.L.dv)[(size_t)bh * D + lane * VEC + v];
        const int j0 = jt * kTile, nvalid = min(kTile, seq_range(a.cu_kv, bh / S.H_kv, S.n_kv, S.total_kv).n - j0);
        if (!rc.wait(k, s_abort, status)) break;
        if (nvalid <= 0) {  // a tile past the end of a shorter packed sequence
            __syncthreads();
            if (threadIdx.x == 0) rc.issue(k + QuantRing<D>::kStages);
            continue;
        }
        const uint16_t *tile = rc.stage(k) + lane * VEC;
        float x[RPW][VEC];
#pragma unroll
        for (int i = 0; i < RPW; ++i) {
            const int r = warp * RPW + i;
            load_row_slice_rt<VEC>(tile + r * D, a.bf16, x[i]);
            if (r >= nvalid) {
#pragma unroll
                for (int v = 0; v < VEC; ++v) x[i][v] = 0.f;
            }
        }
        // the previous tile's store has read the staging tile before it is rewritten
        if (threadIdx.x == 0 && staged) bulk_wait_group_read<0>();
        __syncthreads();  // the stage is in registers: refill it
        if (threadIdx.x == 0) rc.issue(k + QuantRing<D>::kStages);
        if (a.pv16) {
            // FP16 V^T, same key order: per channel, the 8 even keys (16 bytes) at 8w and
            // the 8 odd keys at 64 + 8w
            __half *vt16 = reinterpret_cast<__half *>(a.ws + a.L.vt8) + ((size_t)bh * D + lane * VEC) * S.nk_pad + j0 +
                           warp * (RPW / 2);
#pragma unroll
            for (int v = 0; v < VEC; ++v)
#pragma unroll
                for (int par = 0; par < 2; ++par) {
                    uint32_t w4[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const __half2 h2 = __floats2half2_rn(x[4 * e + par][v], x[4 * e + 2 + par][v]);
                        w4[e] = *reinterpret_cast<const uint32_t *>(&h2);
                    }
                    *reinterpret_cast<uint4 *>(vt16 + (size_t)v * S.nk_pad + par * (kTile / 2)) =
                        make_uint4(w4[0], w4[1], w4[2], w4[3]);
                }
            continue;
        }
        // keys j0 + 16w + i: even i at position 8w + i/2, odd i at 64 + 8w + i/2; channel c's
        // row of the staging tile holds the 128 positions, 16-byte chunk h at (h ^ (c & 7))
        uint8_t *vt8 = a.ws + a.L.vt8 + ((size_t)bh * D + lane * VEC) * S.nk_pad + j0 + warp * (RPW / 2);
#pragma unroll
        for (int v = 0; v < VEC; ++v) {
            uint32_t w[2][2];
            if (dv[v] >= kQuotientMinDelta) {   // the E4M3 codes of the correctly rounded quotients
                const float y = 1.0f / dv[v];
                const float2 y2 = make_float2(y, y), nd2 = make_float2(-dv[v], -dv[v]);
#pragma unroll
                for (int par = 0; par < 2; ++par)
#pragma unroll
                    for (int q = 0; q < 2; ++q)
                        w[par][q] = e4m3x4_codes_rn(x[8 * q + par][v], x[8 * q + 2 + par][v], x[8 * q + 4 + par][v],
                                                    x[8 * q + 6 + par][v], y2, nd2);
            } else {   // a channel of tiny values: IEEE divisions
#pragma unroll
                for (int par = 0; par < 2; ++par)
#pragma unroll
                    for (int q = 0; q < 2; ++q)
                        w[par][q] = pack_e4m3x4(__fdiv_rn(x[8 * q + par][v], dv[v]), __fdiv_rn(x[8 * q + 2 + par][v], dv[v]),
                                                __fdiv_rn(x[8 * q + 4 + par][v], dv[v]),
                                                __fdiv_rn(x[8 * q + 6 + par][v], dv[v]));
            }
            if (staged) {
                const uint32_t c = (uint32_t)(lane * VEC + v), half8 = 8u * (uint32_t)(warp & 1);
                *reinterpret_cast<uint2 *>(vts + sw128_offset(c, (uint32_t)(warp >> 1)) + half8) =
                    make_uint2(w[0][0], w[0][1]);
                *reinterpret_cast<uint2 *>(vts + sw128_offset(c, 4u + (uint32_t)(warp >> 1)) + half8) =
                    make_uint2(w[1][0], w[1][1]);
            } else {
                *reinterpret_cast<uint2 *>(vt8 + (size_t)v * S.nk_pad) = make_uint2(w[0][0], w[0][1]);
                *reinterpret_cast<uint2 *>(vt8 + (size_t)v * S.nk_pad + kTile / 2) = make_uint2(w[1][0], w[1][1]);
            }
        }
        if (staged) {
            fence_proxy_async_smem();   // the tile is read by the tensor store (async proxy)
            __syncthreads();
            if (threadIdx.x == 0) {
                tma_store_2d(&a.tm_vt, vts, j0, bh * D);
                bulk_commit_group();
            }
        }
    }
    if (threadIdx.x == 0 && staged) bulk_wait_group<0>();   // the last stores are done
    if (*s_abort && threadIdx.x == 0) rc.drain(k);
}

// ---------------------------------------------------------------------------
template <int D, bool BF16>
static cudaError_t launch_prepass_d(const PrepassArgs &a, cudaStream_t stream) {
    const Shape &S = a.shape;
    if (a.k || a.v) {
        kv_stats_kernel<D, BF16><<<(unsigned)((size_t)S.n_chunks * S.BH_kv), 256, 0, stream>>>(a);
        kv_finalize_kernel<D><<<S.BH_kv, D, 0, stream>>>(a);
    }
    // persistent grids: two CTAs per SM, or one per work unit if fewer
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const size_t smem = QuantRing<D>::kSmemBytes;
    auto grid_of = [&](int units) { return (unsigned)(units < 2 * sms ? units : 2 * sms); };
    if (a.q) {
        auto kq = a.fp4 ? quant_q_kernel<D, true, BF16> : quant_q_kernel<D, false, BF16>;
        cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        kq<<<grid_of(S.BH * S.Tq), kQuantThreads, smem, stream>>>(a);
    }
    if (a.k) {
        auto kk = a.fp4 ? quant_k_kernel<D, true, BF16> : quant_k_kernel<D, false, BF16>;
        cudaFuncSetAttribute(kk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        kk<<<grid_of(S.BH_kv * S.Tk), kQuantThreads, smem, stream>>>(a);
    }
    if (a.v) {
        const size_t smem_v = QuantVSmem<D>::kBytes;
        cudaFuncSetAttribute(quant_v_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_v);
        quant_v_kernel<D><<<grid_of(S.BH_kv * S.Tk), kQuantThreads, smem_v, stream>>>(a);
    }
    return cudaGetLastError();
}

cudaError_t launch_prepass(const PrepassArgs &a, cudaStream_t stream) {
    if (a.shape.d == 128) return a.bf16 ? launch_prepass_d<128, true>(a, stream) : launch_prepass_d<128, false>(a, stream);
    return a.bf16 ? launch_prepass_d<64, true>(a, stream) : launch_prepass_d<64, false>(a, stream);
}

}  // namespace sage
