// Internal helpers shared by the libmoe CUDA sources.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"

#define MOE_API extern "C" __attribute__((visibility("default")))

namespace moe {

constexpr int kMaxE = 4096;
constexpr int kMaxK = 16;
constexpr int kMaxDim = 8192;

inline cudaStream_t as_cuda(moe_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

// Reports a rejected launch without clearing sticky errors of other work.
inline moe_status launch_status() {
    cudaError_t e = cudaPeekAtLastError();
    if (e != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    return MOE_OK;
}

__device__ __forceinline__ void flag(int32_t *status, int bit) {
    if (status) atomicOr(status, bit);
}

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

inline bool dims_ok(int d, int f) {
    return d > 0 && f > 0 && d % 256 == 0 && f % 256 == 0 && d <= kMaxDim && f <= kMaxDim;
}

}  // namespace moe
