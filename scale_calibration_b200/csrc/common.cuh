// Shared host/device helpers of the calibration library (internal header).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "lh.h"

namespace lh {

// ---------------------------------------------------------------- host side
// Records a detail message for lh_last_error_message() and returns `s`.
lh_status fail(lh_status s, const char* fmt, ...);
// Maps a CUDA error to LH_ERR_CUDA with the error name; LH_OK if none.
lh_status cuda_status(cudaError_t e, const char* what);
// Clears the thread-local message (start of every entry point).
void clear_error();

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline int64_t elem_bytes(lh_dtype t) { return t == LH_BF16 ? 2 : 4; }
inline bool valid_dtype(int t) { return t == LH_BF16 || t == LH_F32; }

// Number of SMs of the current device (cached per device).
int sm_count();

// ---------------------------------------------------------------- device side
__device__ __forceinline__ float bf16_bits_to_float(uint16_t h) {
    return __uint_as_float(static_cast<uint32_t>(h) << 16);
}

}  // namespace lh
