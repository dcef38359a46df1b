// msa_decode_fused_noalloc: the fused decode step for callers that cannot
// allocate device memory.
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
// is looked up once per device, on the first call made with that device
// current; make that first call before capturing any stream.
#include <mutex>

#include "msa_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 8u << 20;  // 8 MiB

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mutex;
void *g_noalloc_ptr[64] = {};

}  // namespace

extern "C" MSA_API msa_status_t msa_decode_fused_noalloc(const msa_params_t *params, const void *q, const void *q_idx,
                                                         const void *k_cache, const void *v_cache, const void *k_idx,
                                                         void *o, int32_t *ids_out, float *lse, msa_stream_t stream) {
    size_t need = 0;
    const msa_status_t st = msa::decode_fused_scratch_bytes(params, &need);  // also checks params and device
    if (st != MSA_OK) return st;
    if (need > kNoAllocScratchBytes)
        return msa::set_error(MSA_ERR_WORKSPACE,
                              "msa_decode_fused_noalloc: these shapes need %zu bytes of scratch but its fixed scratch "
                              "holds %zu; call msa_decode_fused with a workspace instead",
                              need, kNoAllocScratchBytes);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return msa::set_error(MSA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= 64) return msa::set_error(MSA_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
    void *scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_noalloc_mutex);
        if (g_noalloc_ptr[dev] == nullptr) {
            // the array's device address on this device (the host-side symbol is not one)
            void *ptr = nullptr;
            e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
            if (e != cudaSuccess || ptr == nullptr)
                return msa::set_error(MSA_ERR_CUDA, "cudaGetSymbolAddress of the fixed scratch: %s",
                                      cudaGetErrorString(e));
            g_noalloc_ptr[dev] = ptr;
        }
        scratch = g_noalloc_ptr[dev];
    }
    // nothing in the scratch has to start at zero: the scan rewrites the piece table and the
    // candidates and zeroes the split counters at the start of every call
    return msa_decode_fused(params, q, q_idx, k_cache, v_cache, k_idx, o, ids_out, lse, scratch, kNoAllocScratchBytes,
                            stream);
}
