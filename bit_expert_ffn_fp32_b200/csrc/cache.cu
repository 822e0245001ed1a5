// Expert-cache lookup: which routed pairs have their expert in the HBM pool.
//
// Hot experts live in a GPU-memory cache ("5070ti16g单卡跑qwen 3.8 flash next 新方案最高
// 90t/s Hermes调用60t/s", section "为什么从 18t/s 变成 60-90t/s"); the rest are computed
// by the CPU ("个人开发者用 AI 十天写出 Strata 引擎，让 12GB 显存跑起 1250 亿参数的 Qwen 3.8
// Flash Next", section "命中率七成，代价是答案会变"). Residency is per expert, so the
// misses of a non-resident expert are exactly its segment of the sorted
// permutation; the miss list is those segments, experts ascending, which is
// (expert, token) order.
#include <algorithm>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kThreads = 1024;

__global__ void __launch_bounds__(kThreads)
    cache_lookup_kernel(const int32_t *slot_of, int num_slots, int layer, const int32_t *topk_idx,
                        const float *topk_w, const int32_t *offsets, const int32_t *sorted_tok,
                        const int32_t *sorted_j, int T, int k, int E, int32_t *slot_of_pair, moe_miss *miss,
                        int32_t *miss_count, int miss_cap, int32_t *expert_counts, int32_t *status) {
    __shared__ int s_mbase[kMaxE];
    __shared__ int s_warp[32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // per-thread run of experts; misses per expert = its count if not resident
    const int per = (E + kThreads - 1) / kThreads;
    const int e0 = threadIdx.x * per;
    int sum = 0;
    for (int i = 0; i < per; ++i) {
        const int e = e0 + i;
        if (e < E) {
            const int sl = slot_of[e];
            const bool bad = sl < -1 || sl >= num_slots;
            if (bad && blockIdx.x == 0) flag(status, MOE_DEV_BAD_SLOT);
            const int m = (sl < 0 || bad) ? offsets[e + 1] - offsets[e] : 0;
            s_mbase[e] = m;
            sum += m;
        }
    }
    // exclusive scan of per-thread sums
    int x = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = s_warp[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        s_warp[lane] = w;
    }
    __syncthreads();
    int base = (warp > 0 ? s_warp[warp - 1] : 0) + x - sum;
    const int total = s_warp[31];
    for (int i = 0; i < per; ++i) {
        const int e = e0 + i;
        if (e < E) {
            const int m = s_mbase[e];
            s_mbase[e] = base;
            base += m;
        }
    }
    if (threadIdx.x == 0 && blockIdx.x == 0) {
        *miss_count = total;
        if (total > miss_cap) flag(status, MOE_DEV_MISS_OVERFLOW);
    }
    __syncthreads();
    const int n = T * k;
    for (int s = blockIdx.x * kThreads + threadIdx.x; s < n; s += gridDim.x * kThreads) {
        const int t = sorted_tok[s], j = sorted_j[s];
        const int p = t * k + j;
        const int e = topk_idx[p];
        if (e < 0 || e >= E) {
            flag(status, MOE_DEV_BAD_INDEX);
            slot_of_pair[p] = -1;
            continue;
        }
        if (expert_counts) atomicAdd(expert_counts + e, 1);
        const int sl = slot_of[e];
        const bool resident = sl >= 0 && sl < num_slots;
        slot_of_pair[p] = resident ? sl : -1;
        if (!resident) {
            const int mi = s_mbase[e] + (s - offsets[e]);
            if (mi < miss_cap) {
                moe_miss r;
                r.layer = layer;
                r.expert = e;
                r.token = t;
                r.j = j;
                r.gate = topk_w ? topk_w[p] : 0.0f;
                miss[mi] = r;
            }
        }
    }
}

}  // namespace
}  // namespace moe

using namespace moe;

MOE_API moe_status moe_cache_lookup(const int32_t *slot_of, int32_t num_slots, int32_t layer, const int32_t *topk_idx,
                                    const float *topk_w, const int32_t *offsets, const int32_t *sorted_tok,
                                    const int32_t *sorted_j, int T, int k, int E, int32_t *slot_of_pair,
                                    moe_miss *miss, int32_t *miss_count, int32_t miss_cap, int32_t *expert_counts,
                                    int32_t *dev_status, moe_stream_t stream) {
    if (T < 0 || k <= 0 || E <= 0 || num_slots < 0 || miss_cap < 0) return MOE_ERR_INVALID_ARG;
    if (E > kMaxE || k > kMaxK) return MOE_ERR_UNSUPPORTED;
    if (int64_t(T) * k >= (int64_t(1) << 31)) return MOE_ERR_OVERFLOW;
    if (!slot_of || !offsets || !miss_count || (miss_cap > 0 && !miss)) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!topk_idx || !topk_w || !sorted_tok || !sorted_j || !slot_of_pair)) return MOE_ERR_INVALID_ARG;
    // every CTA scans the per-expert miss bases (E values), then handles its pairs
    const int grid = int(std::min<int64_t>((int64_t(T) * k + kThreads - 1) / kThreads, 148));
    cache_lookup_kernel<<<std::max(grid, 1), kThreads, 0, as_cuda(stream)>>>(slot_of, num_slots, layer, topk_idx, topk_w, offsets,
                                                             sorted_tok, sorted_j, T, k, E, slot_of_pair, miss,
                                                             miss_count, miss_cap, expert_counts, dev_status);
    return launch_status();
}
