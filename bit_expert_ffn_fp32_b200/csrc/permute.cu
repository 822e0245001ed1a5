// Stable token -> expert permutation (counting sort by expert id).
//
// Pairs p = t*k + j are ordered by (expert, p). Tiles of kTile tokens are
// counted independently (histogram), a single CTA turns the per-tile counts
// into per-(tile, expert) starting positions, and each tile then places its
// pairs token by token, so the order inside an expert is the token order with
// no dependence on atomic ordering. Small inputs (one tile) use one fused CTA.
#include "common.cuh"

namespace moe {
namespace {

constexpr int kTile = 64;      // tokens per tile
constexpr int kThreads = 1024;

// Block-wide exclusive scan of one value per thread (kThreads threads).
__device__ int block_exclusive_scan(int v, int *s_warp, int &total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = lane < (kThreads / 32) ? s_warp[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        s_warp[lane] = w;  // inclusive warp totals
    }
    __syncthreads();
    const int before = (warp > 0 ? s_warp[warp - 1] : 0) + x - v;
    total = s_warp[kThreads / 32 - 1];
    __syncthreads();
    return before;
}

// Offsets, counts and the active list from per-expert counts held in s_cnt.
// Each thread owns experts [tid*per, tid*per+per).
__device__ void counts_to_offsets(const int *s_cnt, int E, int32_t *counts, int32_t *offsets, int32_t *active,
                                  int *s_warp) {
    const int per = (E + kThreads - 1) / kThreads;
    const int e0 = threadIdx.x * per;
    int sum = 0, nact = 0;
    for (int i = 0; i < per; ++i) {
        const int e = e0 + i;
        if (e < E) {
            sum += s_cnt[e];
            nact += s_cnt[e] > 0;
        }
    }
    int tot, tot_act;
    int base = block_exclusive_scan(sum, s_warp, tot);
    int abase = block_exclusive_scan(nact, s_warp, tot_act);
    for (int i = 0; i < per; ++i) {
        const int e = e0 + i;
        if (e < E) {
            counts[e] = s_cnt[e];
            offsets[e] = base;
            base += s_cnt[e];
            if (s_cnt[e] > 0) active[1 + abase++] = e;
        }
    }
    if (threadIdx.x == 0) {
        offsets[E] = tot;
        active[0] = tot_act;
    }
}

// Places the pairs of tokens [t0, t1) in token order; s_base[e] = next position of e.
// Runs on warp 0 only; idx_tile holds the tile's expert ids (shared memory).
__device__ void place_tokens(const int32_t *idx_tile, int t0, int t1, int k, int E, int *s_base, int32_t *sorted_tok,
                             int32_t *sorted_j, int32_t *inv, int32_t *status) {
    const int lane = threadIdx.x & 31;
    for (int t = t0; t < t1; ++t) {
        const bool on = lane < k;
        int e = on ? idx_tile[(t - t0) * k + lane] : -1;
        const bool valid = on && e >= 0 && e < E;
        if (on && !valid) flag(status, MOE_DEV_BAD_INDEX);
        const unsigned vmask = __ballot_sync(0xffffffffu, valid);
        const unsigned peers = __match_any_sync(0xffffffffu, valid ? e : -1 - lane);
        if (valid) {
            const unsigned same = peers & vmask;
            if (__popc(same) > 1) flag(status, MOE_DEV_BAD_INDEX);
            const int rank = __popc(same & ((1u << lane) - 1));
            const int pos = s_base[e] + rank;
            sorted_tok[pos] = t;
            sorted_j[pos] = lane;
            inv[size_t(t) * k + lane] = pos;
        }
        __syncwarp();
        if (valid) {
            const unsigned same = peers & vmask;
            if ((same & ((1u << lane) - 1)) == 0) s_base[e] += __popc(same);
        }
        __syncwarp();
    }
}

// Single-CTA path: T <= kTile.
__global__ void __launch_bounds__(kThreads)
    permute_small_kernel(const int32_t *idx, int T, int k, int E, int32_t *counts, int32_t *offsets,
                         int32_t *sorted_tok, int32_t *sorted_j, int32_t *inv, int32_t *active, int32_t *status) {
    __shared__ int s_cnt[kMaxE];
    __shared__ int s_warp[32];
    for (int e = threadIdx.x; e < E; e += kThreads) s_cnt[e] = 0;
    __syncthreads();
    for (int p = threadIdx.x; p < T * k; p += kThreads) {
        const int e = idx[p];
        if (e >= 0 && e < E) atomicAdd(&s_cnt[e], 1);
    }
    __syncthreads();
    counts_to_offsets(s_cnt, E, counts, offsets, active, s_warp);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += kThreads) s_cnt[e] = offsets[e];
    __shared__ int s_idx[kTile * kMaxK];
    for (int i = threadIdx.x; i < T * k; i += kThreads) s_idx[i] = idx[i];
    __syncthreads();
    if (threadIdx.x < 32) place_tokens(s_idx, 0, T, k, E, s_cnt, sorted_tok, sorted_j, inv, status);
}

// Multi-tile path, step 1: per-tile histograms into ws[tile][E].
__global__ void __launch_bounds__(256) permute_hist_kernel(const int32_t *idx, int T, int k, int E, int32_t *ws) {
    __shared__ int s_cnt[kMaxE];
    for (int e = threadIdx.x; e < E; e += blockDim.x) s_cnt[e] = 0;
    __syncthreads();
    const int t0 = blockIdx.x * kTile, t1 = min(T, t0 + kTile);
    for (int p = t0 * k + threadIdx.x; p < t1 * k; p += blockDim.x) {
        const int e = idx[p];
        if (e >= 0 && e < E) atomicAdd(&s_cnt[e], 1);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) ws[size_t(blockIdx.x) * E + e] = s_cnt[e];
}

// Step 2: per-expert scan over tiles (ws becomes each tile's start inside the
// expert), then offsets / counts / active list.
__global__ void __launch_bounds__(kThreads)
    permute_scan_kernel(int ntiles, int E, int32_t *ws, int32_t *counts, int32_t *offsets, int32_t *active) {
    __shared__ int s_cnt[kMaxE];
    __shared__ int s_warp[32];
    constexpr int kBatch = 16;  // tiles whose counts are loaded together (one L2 round trip)
    for (int e = threadIdx.x; e < E; e += kThreads) {
        int run = 0;
        for (int t0 = 0; t0 < ntiles; t0 += kBatch) {
            int h[kBatch];
#pragma unroll
            for (int j = 0; j < kBatch; ++j) h[j] = t0 + j < ntiles ? ws[size_t(t0 + j) * E + e] : 0;
#pragma unroll
            for (int j = 0; j < kBatch; ++j) {
                if (t0 + j < ntiles) ws[size_t(t0 + j) * E + e] = run;
                run += h[j];
            }
        }
        s_cnt[e] = run;
    }
    __syncthreads();
    counts_to_offsets(s_cnt, E, counts, offsets, active, s_warp);
}

// Step 3: each tile places its pairs.
__global__ void __launch_bounds__(128)
    permute_scatter_kernel(const int32_t *idx, int T, int k, int E, const int32_t *ws, const int32_t *offsets,
                           int32_t *sorted_tok, int32_t *sorted_j, int32_t *inv, int32_t *status) {
    __shared__ int s_base[kMaxE];
    __shared__ int s_idx[kTile * kMaxK];
    for (int e = threadIdx.x; e < E; e += blockDim.x) s_base[e] = offsets[e] + ws[size_t(blockIdx.x) * E + e];
    const int t0 = blockIdx.x * kTile, t1 = min(T, t0 + kTile);
    for (int i = threadIdx.x; i < (t1 - t0) * k; i += blockDim.x) s_idx[i] = idx[size_t(t0) * k + i];
    __syncthreads();
    if (threadIdx.x < 32) place_tokens(s_idx, t0, t1, k, E, s_base, sorted_tok, sorted_j, inv, status);
}

}  // namespace
}  // namespace moe

using namespace moe;

MOE_API size_t moe_permute_workspace_bytes(int T, int k, int E) {
    if (T <= kTile || E <= 0) return 0;
    return size_t((T + kTile - 1) / kTile) * size_t(E) * sizeof(int32_t);
}

MOE_API moe_status moe_permute(const int32_t *topk_idx, int T, int k, int E, int32_t *counts, int32_t *offsets,
                               int32_t *sorted_tok, int32_t *sorted_j, int32_t *inv, int32_t *active, void *ws,
                               size_t ws_bytes, int32_t *dev_status, moe_stream_t stream) {
    if (T < 0 || k <= 0 || E <= 0) return MOE_ERR_INVALID_ARG;
    if (E > kMaxE || k > kMaxK) return MOE_ERR_UNSUPPORTED;
    if (int64_t(T) * k >= (int64_t(1) << 31)) return MOE_ERR_OVERFLOW;
    if (!counts || !offsets || !active) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = as_cuda(stream);
    if (T == 0) {
        // Nothing routed: zero counts/offsets/active so later steps see an empty layer.
        cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, s);
        cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), s);
        cudaMemsetAsync(active, 0, sizeof(int32_t), s);
        return launch_status();
    }
    if (!topk_idx || !sorted_tok || !sorted_j || !inv) return MOE_ERR_INVALID_ARG;
    if (T <= kTile) {
        permute_small_kernel<<<1, kThreads, 0, s>>>(topk_idx, T, k, E, counts, offsets, sorted_tok, sorted_j, inv,
                                                    active, dev_status);
        return launch_status();
    }
    const size_t need = moe_permute_workspace_bytes(T, k, E);
    if (!ws || ws_bytes < need) return MOE_ERR_WORKSPACE;
    const int ntiles = (T + kTile - 1) / kTile;
    int32_t *w = static_cast<int32_t *>(ws);
    permute_hist_kernel<<<ntiles, 256, 0, s>>>(topk_idx, T, k, E, w);
    permute_scan_kernel<<<1, kThreads, 0, s>>>(ntiles, E, w, counts, offsets, active);
    permute_scatter_kernel<<<ntiles, 128, 0, s>>>(topk_idx, T, k, E, w, offsets, sorted_tok, sorted_j, inv,
                                                  dev_status);
    return launch_status();
}
