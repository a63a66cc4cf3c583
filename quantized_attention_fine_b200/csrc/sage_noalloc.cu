// sage_noalloc.cu -- sage_attn_fwd_noalloc: the whole forward without a
// caller-supplied workspace.  Its scratch (INT8/FP8 codes, scales, dS, the status
// block) lives in one file-scope device array, held on every GPU where the
// library's device code is loaded until the process exits.
//
// Who needs this: code that must not allocate device memory while it runs, for
// example a plugin whose host application owns every device allocation, or a
// serving loop in which a cudaMalloc (which can synchronize the device and stall
// other streams) is not acceptable.  Such callers still pass their own inputs and
// output; only the scratch comes from here.
//
// Under CUDA's lazy module loading the array is reserved when the library's device
// code is first used on a device: by the first call of this entry point (a call with
// B = 0 does only that), or by any other launch of the library.  That first call
// may allocate and synchronize inside the CUDA runtime, so make it at
// initialisation, before any stream capture.
#include <mutex>

#include "../../include/sage.h"
#include "sage_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 64ull << 20;   // 64 MiB per GPU
constexpr int kMaxDevices = 64;

// Device-side scratch shared by every call on a GPU.  In host code this name is
// only a stand-in for the symbol: its device address comes from
// cudaGetSymbolAddress, once per device.
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
uint8_t *g_noalloc_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up on first use).
sage_status_t noalloc_scratch(uint8_t **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SAGE_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return SAGE_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_addr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return SAGE_ERR_CUDA;
        g_noalloc_addr[dev] = static_cast<uint8_t *>(p);
    }
    *out = g_noalloc_addr[dev];
    return SAGE_OK;
}

}  // namespace

namespace sage {

// The array rounded up to the 1024-byte alignment the workspace layout is built on.
sage_status_t noalloc_workspace(uint8_t **ws, size_t *bytes) {
    uint8_t *base = nullptr;
    const sage_status_t st = noalloc_scratch(&base);
    if (st != SAGE_OK) return st;
    const uintptr_t raw = reinterpret_cast<uintptr_t>(base);
    const uintptr_t aligned = (raw + kWsAlign - 1) & ~(uintptr_t)(kWsAlign - 1);
    *ws = reinterpret_cast<uint8_t *>(aligned);
    *bytes = kNoAllocScratchBytes - (size_t)(aligned - raw);
    return SAGE_OK;
}

}  // namespace sage

extern "C" sage_status_t sage_attn_fwd_noalloc(const void *q, const void *k, const void *v, void *o, int dtype,
                                               int layout, int B, int H, int n_q, int n_kv, int d, int causal,
                                               float sm_scale, const sage_quant_mode_t *mode, void *stream) {
    // The checks of sage_attn_fwd come first, so that an argument error enqueues nothing.
    int plan = sage::kFwdNoop;
    size_t need = 0;
    sage_status_t st = sage::check_fwd_args(q, k, v, o, dtype, layout, B, H, H, n_q, n_kv, d, mode, &plan, &need);
    if (st != SAGE_OK) return st;
    // Looked up even for a call with nothing to do: such a call reserves the array.
    uint8_t *ws = nullptr;
    size_t usable = 0;
    st = sage::noalloc_workspace(&ws, &usable);
    if (st != SAGE_OK) return st;
    if (plan == sage::kFwdRun) {
        // Problems whose workspace would not fit are refused before anything is enqueued.
        if (need > usable) return SAGE_ERR_WORKSPACE;
        // The array keeps the previous call's contents; the status block must start at zero.
        if (cudaMemsetAsync(ws, 0, sage::kStatusBytes, static_cast<cudaStream_t>(stream)) != cudaSuccess)
            return SAGE_ERR_CUDA;
    }
    return sage_attn_fwd(q, k, v, o, dtype, layout, B, H, n_q, n_kv, d, causal, sm_scale, mode, ws, usable, stream);
}

extern "C" sage_status_t sage_noalloc_get_device_status(void *stream, int *code, int *site) {
    if (!code || !site) return SAGE_ERR_INVALID_ARG;
    uint8_t *ws = nullptr;
    size_t usable = 0;
    const sage_status_t st = sage::noalloc_workspace(&ws, &usable);
    if (st != SAGE_OK) return st;
    return sage_get_device_status(ws, stream, code, site);
}
