// Gate-weighted combine plus the always-on shared expert ("个人开发者用 AI 十天写出
// Strata 引擎，让 12GB 显存跑起 1250 亿参数的 Qwen 3.8 Flash Next", section
// "1250 亿参数，每个词只用得上 2%": every token uses its routed experts and one shared
// expert). y[t] = y_shared[t] + sum_j gate[t][j] * y_perm[inv[t*k+j]] over the
// pairs whose expert is resident, j in increasing order.
#include <algorithm>

#include "common.cuh"

namespace moe {
namespace {

__global__ void combine_kernel(const float *__restrict__ y_perm, const int32_t *__restrict__ inv,
                               const float *__restrict__ topk_w, const int32_t *__restrict__ slot_of_pair,
                               const float *__restrict__ y_shared, int T, int k, int d, float *__restrict__ y) {
    const int d4 = d / 4;
    const int64_t n = int64_t(T) * d4;
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
        const int t = int(i / d4), c = int(i % d4);
        float4 acc = y_shared ? reinterpret_cast<const float4 *>(y_shared + int64_t(t) * d)[c]
                              : make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = 0; j < k; ++j) {
            const int p = t * k + j;
            if (slot_of_pair && slot_of_pair[p] < 0) continue;
            const float g = topk_w[p];
            const float4 v = reinterpret_cast<const float4 *>(y_perm + int64_t(inv[p]) * d)[c];
            acc.x = fmaf(g, v.x, acc.x);
            acc.y = fmaf(g, v.y, acc.y);
            acc.z = fmaf(g, v.z, acc.z);
            acc.w = fmaf(g, v.w, acc.w);
        }
        reinterpret_cast<float4 *>(y + int64_t(t) * d)[c] = acc;
    }
}

}  // namespace
}  // namespace moe

using namespace moe;

MOE_API moe_status moe_combine(const float *y_perm, const int32_t *inv, const float *topk_w,
                               const int32_t *slot_of_pair, const float *y_shared, int T, int k, int d, float *y,
                               moe_stream_t stream) {
    if (T < 0 || k <= 0 || d <= 0) return MOE_ERR_INVALID_ARG;
    if (d % 4 || k > kMaxK) return MOE_ERR_UNSUPPORTED;
    if (int64_t(T) * k >= (int64_t(1) << 31)) return MOE_ERR_OVERFLOW;
    if (T == 0) return MOE_OK;
    if (!y_perm || !inv || !topk_w || !y) return MOE_ERR_INVALID_ARG;
    const int64_t n = int64_t(T) * (d / 4);
    const int blocks = int(std::min<int64_t>((n + 255) / 256, 148 * 16));
    combine_kernel<<<blocks, 256, 0, as_cuda(stream)>>>(y_perm, inv, topk_w, slot_of_pair, y_shared, T, k, d, y);
    return launch_status();
}
