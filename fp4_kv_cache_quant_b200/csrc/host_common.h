// host_common.h -- small host-side helpers shared by the library's entry points.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/bdfp4.h"

namespace bdfp4 {

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline bool supported_dims(int d_k, int d_v) { return (d_k == 128 && d_v == 128) || (d_k == 576 && d_v == 512); }

// Last CUDA error the library saw on this thread (for bdfp4_last_error).
void record_cuda_error(cudaError_t e);

// Status of the launches just made on this thread.
inline int launch_status() {
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) return BDFP4_OK;
    record_cuda_error(e);
    return BDFP4_ERR_CUDA;
}

}  // namespace bdfp4
