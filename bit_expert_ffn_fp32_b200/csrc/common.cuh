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

// Prefill path (ffn_tc05.cu): grouped tcgen05 GEMMs for Q2 or Q3 experts. Used
// by moe_expert_ffn_q2/q3 when T*k >= kTcMinPairs; the caller has validated
// arguments.
constexpr int kTcMinPairs = 512;
constexpr int kTcMaxE = 1024;
// Byte offset of the permuted fp16 activations (fp16 [T*k][d]) inside the
// tensor-core path's workspace (after h, fp16 [T*k][f], rounded up to 256 B).
inline size_t tc05_xperm_offset(int T, int k, int f) {
    return (size_t(T) * size_t(k) * size_t(f) * 2 + 255) & ~size_t(255);
}
moe_status tc05_ffn(int fmt, const moe_qpool *W, const int32_t *slot_of, const uint16_t *x, int T, int d, int f, int E,
                    int k, const int32_t *offsets, const int32_t *sorted_tok, const int32_t *sorted_j,
                    const int32_t *active, const float *topk_w, float *out, void *ws, int32_t *dev_status,
                    cudaStream_t stream);

}  // namespace moe
