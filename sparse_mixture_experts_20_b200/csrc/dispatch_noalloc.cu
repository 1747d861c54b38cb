// moe_dispatch_noalloc: moe_dispatch without a caller-provided workspace.
//
// The dispatch kernels need scratch memory for their per-expert token bitmaps
// and word prefix counts.  moe_dispatch takes it from the caller's workspace;
// this entry point takes it from a fixed array in device memory that is part
// of the library image instead, so that a caller which cannot allocate device
// memory can still dispatch.  Every GPU that loads the library holds the
// array (kNoAllocScratchBytes) until the process exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <mutex>
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr size_t kNoAllocScratchBytes = 2u << 20;   // 2 MiB

// Scratch shared by every call of moe_dispatch_noalloc on this device.
static __device__ __align__(256) uint8_t g_dispatch_scratch[kNoAllocScratchBytes];

// Device addresses of g_dispatch_scratch, one per CUDA context.  In host code
// the symbol is a host-side stand-in, not a device address, and each context
// (the device's primary context, a context of the caller's own, the primary
// context recreated after a device reset) loads the library's device image
// at its own address; the cache is keyed on the context's id, which the
// driver never reuses within a process.
struct ScratchEntry {
    unsigned long long ctx_id;
    void* ptr;
};
constexpr int kCacheEntries = 64;
ScratchEntry g_scratch_cache[kCacheEntries] = {};
int g_scratch_cached = 0;
std::mutex g_scratch_mutex;

PFN_cuCtxGetId_v12000 ctx_id_fn() {
    static PFN_cuCtxGetId_v12000 fn = [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<PFN_cuCtxGetId_v12000>(ptr);
        return static_cast<PFN_cuCtxGetId_v12000>(nullptr);
    }();
    return fn;
}

// Device address of g_dispatch_scratch in the calling thread's current
// context, looked up (cudaGetSymbolAddress) the first time this context calls.
cudaError_t scratch_in_current_context(void** out) {
    auto get_id = ctx_id_fn();
    if (!get_id) return cudaErrorNotSupported;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    unsigned long long id = 0;
    const bool have_ctx = get_id(nullptr, &id) == CUDA_SUCCESS;
    if (have_ctx) {
        for (int i = 0; i < kCacheEntries && i < g_scratch_cached; ++i)
            if (g_scratch_cache[i].ctx_id == id) {
                *out = g_scratch_cache[i].ptr;
                return cudaSuccess;
            }
    }
    // first call in this context (or no context current yet: the lookup makes
    // the device's primary context current)
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_dispatch_scratch);
    if (e != cudaSuccess) return e;
    if (!have_ctx && get_id(nullptr, &id) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
    g_scratch_cache[g_scratch_cached % kCacheEntries] = {id, p};
    ++g_scratch_cached;
    *out = p;
    return cudaSuccess;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" int moe_dispatch_noalloc(const moe_config* cfg, const void* x, const int32_t* topk_idx,
                                    int32_t* counts, int32_t* kept, int32_t* offsets, int32_t* slot_row,
                                    int32_t* row_slot, void* x_disp, float* x_disp_scales, void* stream) {
    NvtxRange nvtx("moe_dispatch_noalloc");
    Dims dm;
    const int v = validate(cfg, &dm);
    if (v != MOE_OK) return v;
    if (!x || !topk_idx || !counts || !kept || !offsets || !slot_row || !row_slot || !x_disp)
        return MOE_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(x) & 15u) || (reinterpret_cast<uintptr_t>(x_disp) & 15u))
        return MOE_ERR_INVALID_ARG;
    if (dm.dtype == MOE_FP8_E4M3_BLOCK && !x_disp_scales) return MOE_ERR_INVALID_ARG;
    // bitmap and word bases, each (planes, T/32, N_r) 32-bit words, 256-byte aligned
    const size_t part = (static_cast<size_t>(dm.planes) * dm.t_words * dm.E * 4 + 255) & ~static_cast<size_t>(255);
    if (2 * part > kNoAllocScratchBytes) return MOE_ERR_UNSUPPORTED;
    void* base = nullptr;
    cudaError_t e = scratch_in_current_context(&base);
    if (e == cudaSuccess) {
        // Both regions are fully rewritten by every call: nothing to clear.
        uint32_t* bitmap = static_cast<uint32_t*>(base);
        int32_t* word_base = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(base) + part);
        e = launch_dispatch(dm, x, topk_idx, counts, kept, offsets, slot_row, row_slot, x_disp, x_disp_scales,
                            bitmap, word_base, nullptr, static_cast<cudaStream_t>(stream));
    }
    if (e != cudaSuccess) {
        note_cuda_error(static_cast<int>(e));
        return MOE_ERR_CUDA;
    }
    return MOE_OK;
}
