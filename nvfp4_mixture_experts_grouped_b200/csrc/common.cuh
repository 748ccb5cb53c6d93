// common.cuh -- shared host/device plumbing of the sm_100a MoE library.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/nvfp4moe.h"

namespace nvfp4moe {

// ---------------------------------------------------------------------------
// Host-side error reporting
// ---------------------------------------------------------------------------
void set_error(const char* fmt, ...);

#define NVFP4MOE_CHECK_LAUNCH(what)                                                            \
    do {                                                                                        \
        cudaError_t _e = cudaGetLastError();                                                    \
        if (_e != cudaSuccess) {                                                                \
            ::nvfp4moe::set_error("%s: %s", what, cudaGetErrorString(_e));                      \
            return NVFP4MOE_ERR_CUDA;                                                           \
        }                                                                                       \
    } while (0)

#define NVFP4MOE_CUDA(call)                                                                    \
    do {                                                                                        \
        cudaError_t _e = (call);                                                                \
        if (_e != cudaSuccess) {                                                                \
            ::nvfp4moe::set_error("%s: %s", #call, cudaGetErrorString(_e));                     \
            return NVFP4MOE_ERR_CUDA;                                                           \
        }                                                                                       \
    } while (0)

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }

// Device error word, a set of bits (never trapped): DEV_ERR_TIMEOUT from bounded
// waits that give up; DEV_ERR_BAD_ROUTING from precomputed routing that names an
// expert outside [0, E) or one expert twice for a token.  Only the timeout bit
// makes the other waits of a kernel give up too.
enum : int32_t { DEV_ERR_NONE = 0, DEV_ERR_TIMEOUT = 1, DEV_ERR_BAD_ROUTING = 2 };
int32_t* device_error_word();  // device address of the word (current device and context)
// The driver's id of the calling thread's current CUDA context (unique for the
// process's lifetime, unlike the context handle, which a new context can reuse);
// 0 if there is none or the driver does not provide the calls.
unsigned long long current_context_id();

// Number of SMs of the current device (cached per device).
int num_sms();

// ---------------------------------------------------------------------------
// Device helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ int warp_id() { return threadIdx.x >> 5; }
__device__ __forceinline__ int lane_id() { return threadIdx.x & 31; }

}  // namespace nvfp4moe
