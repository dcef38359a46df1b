// msa_decode_fused_noalloc: the fused decode step for callers that cannot
// allocate device memory, and the status calls of its fixed scratch.
//
// Some callers only ever receive their input and output buffers: plugin or
// foreign-function hosts whose calling convention has no slot for a scratch
// buffer, or serving loops that reserve all device memory at start-up and
// forbid allocation afterwards.  They cannot provide the workspace that
// msa_decode_fused needs, so this entry point takes its scratch from a
// fixed array in device memory that belongs to the library itself.
//
// The array lives for as long as the library is loaded, on every GPU that
// loads it (kNoAllocScratchBytes each).  All calls share it: two calls whose
// work overlaps on the GPU (different streams, or different host threads on
// the same device) race on it and must be ordered by the caller.  Its address
// is looked up on the first call made with a device current (and again when
// that device's context has been replaced, e.g. after cudaDeviceReset); make
// that first call before capturing any stream.
#include <cudaTypedefs.h>

#include <mutex>

#include "msa_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 8u << 20;  // 8 MiB

// Its head (status word, wait limit, the scan's work counters) must start at zero: a __device__
// array is zero-filled when the module is loaded, every scan returns its counters to zero when it
// ends, and msa_noalloc_clear_status resets the head after a call that did not end normally.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

struct ScratchSlot {
    unsigned long long ctx_id = 0;  // driver id of the context the address belongs to
    void *ptr = nullptr;
};

std::mutex g_noalloc_mutex;
ScratchSlot g_noalloc_slot[64];

// Unique id of the calling thread's current context (0 if the driver cannot tell).
unsigned long long current_context_id() {
    static PFN_cuCtxGetCurrent_v4000 get_cur = nullptr;
    static PFN_cuCtxGetId_v12000 get_id = nullptr;
    static bool looked_up = false;
    if (!looked_up) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_cur = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
        looked_up = true;
    }
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_cur == nullptr || get_id == nullptr || get_cur(&ctx) != CUDA_SUCCESS || ctx == nullptr ||
        get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

// Device address of the fixed scratch on the current device (the host-side
// symbol is not one).
msa_status_t noalloc_scratch(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return msa::set_error(MSA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= 64) return msa::set_error(MSA_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
    // the runtime sets up the device's primary context here (if it has not yet), so that it has an id
    e = cudaSetDevice(dev);
    if (e != cudaSuccess) return msa::set_error(MSA_ERR_CUDA, "cudaSetDevice: %s", cudaGetErrorString(e));
    const unsigned long long ctx = current_context_id();
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    ScratchSlot &slot = g_noalloc_slot[dev];
    if (slot.ptr == nullptr || slot.ctx_id != ctx) {
        void *ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (e != cudaSuccess || ptr == nullptr)
            return msa::set_error(MSA_ERR_CUDA, "cudaGetSymbolAddress of the fixed scratch: %s", cudaGetErrorString(e));
        slot.ptr = ptr;
        slot.ctx_id = ctx;
    }
    *out = slot.ptr;
    return MSA_OK;
}

}  // namespace

extern "C" MSA_API msa_status_t msa_decode_fused_noalloc(const msa_params_t *params, const void *q, const void *q_idx,
                                                         const void *k_cache, const void *v_cache, const void *k_idx,
                                                         void *o, int32_t *ids_out, float *lse, msa_stream_t stream) {
    size_t need = 0;
    msa_status_t st = msa::decode_fused_scratch_bytes(params, &need);  // also checks params and device
    if (st != MSA_OK) return st;
    if (need > kNoAllocScratchBytes)
        return msa::set_error(MSA_ERR_WORKSPACE,
                              "msa_decode_fused_noalloc: these shapes need %zu bytes of scratch but its fixed scratch "
                              "holds %zu; call msa_decode_fused with a workspace instead",
                              need, kNoAllocScratchBytes);
    void *scratch = nullptr;
    if ((st = noalloc_scratch(&scratch)) != MSA_OK) return st;
    // the piece table, candidate lists and split counters are rewritten by every call; the head
    // is zero unless a call timed out (see msa_noalloc_get_status / msa_noalloc_clear_status)
    return msa_decode_fused(params, q, q_idx, k_cache, v_cache, k_idx, o, ids_out, lse, scratch, kNoAllocScratchBytes,
                            stream);
}

extern "C" MSA_API msa_status_t msa_noalloc_get_status(int *status, msa_stream_t stream) {
    if (status == nullptr) return msa::set_error(MSA_ERR_INVALID_ARG, "status is NULL");
    void *scratch = nullptr;
    const msa_status_t st = noalloc_scratch(&scratch);
    if (st != MSA_OK) return st;
    return msa_get_device_status(scratch, status, stream);
}

extern "C" MSA_API msa_status_t msa_noalloc_clear_status(msa_stream_t stream) {
    void *scratch = nullptr;
    const msa_status_t st = noalloc_scratch(&scratch);
    if (st != MSA_OK) return st;
    return msa_clear_device_status(scratch, stream);
}
