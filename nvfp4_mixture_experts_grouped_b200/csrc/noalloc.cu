// noalloc.cu -- moe_permute_noalloc: the token permutation for callers that
// cannot allocate device memory.
//
// Its scratch is a file-scope static device array instead of a caller-provided
// workspace.  In host code `g_noalloc_permute_scratch` is only a host-side
// stand-in for the device symbol, never a device address: handing it to a
// kernel would fault, or silently touch the wrong memory where the GPU can reach
// host memory.  The device address is therefore looked up with the device
// current, through cudaGetSymbolAddress, and cached per device together with
// the id of the CUDA context it belongs to: a new context on the device (after
// cudaDeviceReset, for instance) holds the array at a new address, so a context
// id that no longer matches makes the next call look the address up again.
#include <cuda.h>

#include <mutex>

#include "common.cuh"
#include "moe_internal.cuh"

namespace nvfp4moe {

// Every GPU that loads the library holds this array until the process exits.
static __device__ __align__(256) uint8_t g_noalloc_permute_scratch[NVFP4MOE_NOALLOC_SCRATCH_BYTES];

static void* noalloc_scratch_address(nvfp4moe_status* st) {
    static std::mutex mu;
    static void* cache[64] = {};
    static unsigned long long cache_ctx[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        set_error("moe_permute_noalloc: no usable current CUDA device");
        *st = NVFP4MOE_ERR_CUDA;
        return nullptr;
    }
    const unsigned long long ctx = current_context_id();
    std::lock_guard<std::mutex> lk(mu);
    if (!cache[dev] || ctx == 0 || cache_ctx[dev] != ctx) {
        // also makes the device's primary context current if no context was
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_permute_scratch);
        if (e != cudaSuccess || !p) {
            set_error("moe_permute_noalloc: cudaGetSymbolAddress of the scratch array failed on device %d: %s", dev,
                      cudaGetErrorString(e));
            *st = NVFP4MOE_ERR_CUDA;
            return nullptr;
        }
        cache[dev] = p;
        cache_ctx[dev] = ctx != 0 ? ctx : current_context_id();
    }
    *st = NVFP4MOE_OK;
    return cache[dev];
}

}  // namespace nvfp4moe

using namespace nvfp4moe;

extern "C" nvfp4moe_status moe_permute_noalloc(const int32_t* topk_ids, int32_t T, int32_t E, int32_t top_k,
                                               int32_t pad, int32_t* counts_out, int32_t* pad_offsets_out,
                                               int32_t* row_of_pair_out, void* stream) {
    const size_t need = moe_permute_workspace_size(T, E, top_k, pad);
    if (need == 0 || need > NVFP4MOE_NOALLOC_SCRATCH_BYTES) {
        set_error("moe_permute_noalloc: T=%d, E=%d, top_k=%d, pad=%d need %zu bytes of scratch, above the fixed %u "
                  "(T*top_k <= 65536 with E <= 256 always fits); use moe_permute with a workspace instead",
                  T, E, top_k, pad, need, (unsigned)NVFP4MOE_NOALLOC_SCRATCH_BYTES);
        return NVFP4MOE_ERR_UNSUPPORTED_SHAPE;
    }
    nvfp4moe_status st;
    void* scratch = noalloc_scratch_address(&st);
    if (!scratch) return st;
    // The permutation kernels write every scratch word they later read (chunk
    // counts, offsets, tile list), so nothing has to be cleared between calls.
    return moe_permute(topk_ids, T, E, top_k, pad, counts_out, pad_offsets_out, row_of_pair_out, scratch,
                       NVFP4MOE_NOALLOC_SCRATCH_BYTES, stream);
}
