// One whole MoE layer for a few tokens (decode, MTP verify) in one
// cooperative launch.
//
// Per token the router scores the layer's experts, the top k (10 of 512 in
// "个人开发者用 AI 十天写出 Strata 引擎，让 12GB 显存跑起 1250 亿参数的 Qwen 3.8 Flash
// Next", section "1250 亿参数，每个词只用得上 2%") run as SwiGLU experts on packed
// 2/3-bit weights, hot experts are read from an HBM pool and the rest are
// reported as misses ("5070ti16g单卡跑qwen 3.8 flash next 新方案最高90t/s Hermes
// 调用60t/s", section "为什么从 18t/s 变成 60-90t/s"), and the always-on shared expert
// is added. With T <= 8 tokens the layer reads ~20 MB and does little arithmetic,
// so it is bound by HBM and by latency; this kernel keeps every SM streaming:
//
//  A  (no routing needed)  router logits for all experts, the shared expert's
//     gate/up, zeroing of y -- all CTAs at once;
//     grid barrier (logits complete);
//  B  every CTA computes the top-k, gates and permutation itself from the
//     logits in L2 (no second barrier), CTA 0 writes them out, and every CTA
//     issues L2 bulk prefetches for the expert rows its later tasks read, so
//     HBM streams the selected experts at once;
//  C  routed gate/up tasks (expert, 16-row group): h = silu(Wg x) * (Wu x) into
//     scratch, then a per-expert completion counter;
//  D  down tasks (expert or shared, 16-row group) wait for their expert's
//     counter, compute Wd h and add gate * y_e into y with atomics.
//
// Every wait is bounded (MOE_DEV_TIMEOUT after 100 ms) and the last CTA to
// leave resets the counters, so the workspace stays zeroed between launches.
#include <algorithm>
#include <math.h>
#include <mutex>

#include "common.cuh"
#include "layout.h"
#include "mma_q.cuh"

// Optional phase timestamps (build with -DMOE_DECODE_TRACE): thread 0 of every
// CTA records %globaltimer at each phase boundary into moe_decode_trace.
#ifdef MOE_DECODE_TRACE
__device__ unsigned long long moe_decode_trace[4096 * 32];
#define TRACE(i)                                                                                      \
    do {                                                                                              \
        if (threadIdx.x == 0) {                                                                       \
            unsigned long long t_;                                                                    \
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                                    \
            moe_decode_trace[blockIdx.x * 32 + (i)] = t_;                                             \
            moe_decode_trace[blockIdx.x * 32 + 16 + (i)] = clock64();                                 \
        }                                                                                             \
    } while (0)
#define TRACEW(i)                                                                                     \
    do {                                                                                              \
        if ((threadIdx.x & 31) == 0) {                                                                \
            unsigned long long t_;                                                                    \
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                                    \
            moe_decode_trace[blockIdx.x * 32 + (i)] = t_;                                             \
            moe_decode_trace[blockIdx.x * 32 + 16 + (i)] = clock64();                                 \
        }                                                                                             \
    } while (0)
#else
#define TRACE(i) \
    do {         \
    } while (0)
#define TRACEW(i) \
    do {          \
    } while (0)
#endif

namespace moe {
namespace {

#ifndef MOE_DECODE_CTAS_PER_SM
#define MOE_DECODE_CTAS_PER_SM 1
#endif
constexpr int kCtasPerSm = MOE_DECODE_CTAS_PER_SM;  // resident CTAs per SM (register budget)
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxTokDec = 8;
constexpr int kMaxEDec = 512;
constexpr int kMaxPairs = kMaxTokDec * kMaxK;  // 128
constexpr int kSharedIdx = kMaxPairs;         // done[] slot of the shared expert
constexpr int kMaxDimDec = 2048;
constexpr int kCandMax = 64;  // candidates ranked in shared memory; more take the round-based path
constexpr unsigned long long kWaitNs = 100ull * 1000 * 1000;

struct DecodeParams {
    const uint8_t *pool;
    int64_t slot_bytes;
    int num_slots;
    const int32_t *slot_of;
    int shared_slot;
    int layer;
    const uint16_t *x;
    const float *Wr;
    const float *bias;
    int T, d, f, E, k;
    float *logits;
    int32_t *topk_idx;
    float *topk_w;
    int32_t *counts, *offsets, *sorted_tok, *sorted_j, *inv, *active, *slot_of_pair;
    moe_miss *miss;
    int32_t *miss_count;
    int miss_cap;
    float *y;
    int32_t *status;
    unsigned *ctr;   // [0] barrier arrivals, [1] CTAs finished
    unsigned *done;  // [kMaxPairs + 1] gate/up tasks finished per resident expert
    float *h;        // [(T*k + T)][f]: sorted pair rows, then shared-expert rows
    MatGeom gate, up, down;
};

struct Smem {
    float xs[kMaxDimDec / 64][kMaxTokDec];  // block sums of x per token
    float red[kWarps][2][4][32];            // split-K partials of gate/up
    int slot[kMaxEDec];                     // this layer's expert -> slot table
    int idx[kMaxTokDec][kMaxK];
    float w[kMaxTokDec][kMaxK];
    int pair_e[kMaxPairs];                  // expert of sorted pair s
    int s_tok[kMaxPairs], s_j[kMaxPairs];   // sorted pairs
    int inv[kMaxPairs];
    int act_e[kMaxPairs], act_beg[kMaxPairs], act_cnt[kMaxPairs], act_slot[kMaxPairs], act_mbase[kMaxPairs];
    int res[kMaxPairs];                     // active index of each resident expert
    float hsb[1024 / 64][kMaxTokDec];       // block sums of the staged h rows
    uint64_t cand[kMaxTokDec][kCandMax];    // top-k candidates per token
    float sel_v[kMaxTokDec][kMaxK];
    int sel_id[kMaxTokDec][kMaxK];
    unsigned first_mask[kMaxPairs / 32];    // pair s starts a new expert
    int nact, nres, nmiss;
    int ok, last;
};

__device__ __forceinline__ unsigned long long globaltimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ unsigned ld_acquire(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Spin until *p >= target or the time limit; false (and MOE_DEV_TIMEOUT) on timeout.
__device__ bool wait_geq(const unsigned *p, unsigned target, int32_t *status) {
    if (ld_acquire(p) >= target) return true;
    const unsigned long long t0 = globaltimer();
    while (ld_acquire(p) < target) {
        if (globaltimer() - t0 > kWaitNs) {
            flag(status, MOE_DEV_TIMEOUT);
            return false;
        }
        __nanosleep(32);
    }
    return true;
}

// Order-preserving key of an fp32 logit: larger logit -> larger key; +0 and -0
// share one key; 0 is reserved for "no candidate" (NaN, taken, out of range).
__device__ __forceinline__ uint32_t logit_key(float v) {
    if (v != v) return 0u;
    if (v == 0.f) v = 0.f;
    const uint32_t u = __float_as_uint(v);
    const uint32_t k = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return k == 0u ? 1u : k;
}

// Router logits (fixed fp32 order, see moe.h). The 16 chunk loads of a row are
// issued before the activations are staged, so the two overlap.
constexpr int kRouterChunks = kMaxDimDec / 128;  // 16

__device__ __forceinline__ void router_load(const DecodeParams &p, int e, int lane, float4 (&wv)[kRouterChunks]) {
    const float *w = p.Wr + size_t(e) * p.d + 4 * lane;
#pragma unroll
    for (int u = 0; u < kRouterChunks; ++u)
        if (u < p.d / 128) wv[u] = __ldg(reinterpret_cast<const float4 *>(w + 128 * u));
}

template <int NT>
__device__ void router_row(const DecodeParams &p, const uint16_t *sx, int e, int lane,
                           const float4 (&wv)[kRouterChunks]) {
    float acc[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[t] = 0.f;
#pragma unroll
    for (int u = 0; u < kRouterChunks; ++u) {
        if (u >= p.d / 128) break;
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            if (t < p.T) {
                const uint2 xv = *reinterpret_cast<const uint2 *>(sx + size_t(t) * p.d + 128 * u + 4 * lane);
                float a = acc[t];
                a = __fmaf_rn(bf16_lo(xv.x), wv[u].x, a);
                a = __fmaf_rn(bf16_hi(xv.x), wv[u].y, a);
                a = __fmaf_rn(bf16_lo(xv.y), wv[u].z, a);
                a = __fmaf_rn(bf16_hi(xv.y), wv[u].w, a);
                acc[t] = a;
            }
        }
    }
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) acc[t] = __fadd_rn(acc[t], __shfl_xor_sync(0xffffffffu, acc[t], o));
    if (lane == 0) {
        const float b = p.bias ? p.bias[e] : 0.f;
        for (int t = 0; t < p.T; ++t) {
            const float v = p.bias ? __fadd_rn(acc[t], b) : acc[t];
            if (!isfinite(v)) flag(p.status, MOE_DEV_NONFINITE);
            p.logits[size_t(t) * p.E + e] = v;
        }
    }
}

// Gate/up of one 16-row group for up to 8 tokens of one expert into h rows.
// tok[n] = token index (for x and xs), hrow0 + n = scratch row. Whole CTA;
// every warp loads all of its weight tiles before computing.
template <int FMT>
__device__ void gateup_task(const DecodeParams &p, Smem &s, const uint16_t *sx, const uint8_t *rec, int rg,
                            int ntok, const int *tok, int hrow0) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int NQ = p.d / 256;
    float ag[4] = {0.f, 0.f, 0.f, 0.f}, au[4] = {0.f, 0.f, 0.f, 0.f};
    const uint16_t *xrow = g < ntok ? sx + size_t(tok[g]) * p.d : nullptr;
    const int t0 = 2 * t < ntok ? tok[2 * t] : -1, t1 = 2 * t + 1 < ntok ? tok[2 * t + 1] : -1;
    for (int qd = warp; qd < NQ; qd += kWarps) {
        QuadRegs<FMT> qg, qu;
        quad_load<FMT>(rec, p.gate, rg, qd, lane, qg);
        quad_load<FMT>(rec, p.up, rg, qd, lane, qu);
        uint32_t B[4][8];
        build_b_bf16<FMT>(xrow, qd, t, B);
        float xs[4][2];
#pragma unroll
        for (int bq = 0; bq < 4; ++bq) {
            xs[bq][0] = t0 >= 0 ? s.xs[4 * qd + bq][t0] : 0.f;
            xs[bq][1] = t1 >= 0 ? s.xs[4 * qd + bq][t1] : 0.f;
        }
        quad_compute<FMT>(qg, B, xs, ag);
        quad_compute<FMT>(qu, B, xs, au);
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        s.red[warp][0][r][lane] = ag[r];
        s.red[warp][1][r][lane] = au[r];
    }
    __syncthreads();
    if (threadIdx.x < 128) {
        const int L = threadIdx.x >> 2, r = threadIdx.x & 3;
        float A = 0.f, U = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            A += s.red[w][0][r][L];
            U += s.red[w][1][r][L];
        }
        const int row = (L >> 2) + ((r & 2) ? 8 : 0);
        const int n = 2 * (L & 3) + (r & 1);
        if (n < ntok) p.h[size_t(hrow0 + n) * p.f + 16 * rg + row] = A / (1.0f + expf(-A)) * U;
    }
}

// Block sums of the staged activations, one warp per (64-block, token); whole CTA.
__device__ __forceinline__ void stage_xsum(Smem &s, const uint16_t *sx, int NB, int T, int d) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int job = warp; job < NB * T; job += kWarps) {
        const int b = job / T, n = job % T;
        const uint32_t u = *reinterpret_cast<const uint32_t *>(sx + size_t(n) * d + 64 * b + 2 * lane);
        float v = bf16_lo(u) + bf16_hi(u);
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) s.xs[b][n] = v;
    }
}

template <int FMT, int NT>
__global__ void __launch_bounds__(kThreads, kCtasPerSm) decode_layer_kernel(DecodeParams p) {
    extern __shared__ __align__(16) unsigned char dyn[];
    __shared__ Smem s;
    uint16_t *sx = reinterpret_cast<uint16_t *>(dyn);                                        // [T][d] bf16
    float *sh = reinterpret_cast<float *>(dyn + ((size_t(p.T) * p.d * 2 + 15) & ~size_t(15)));  // [8][f] h
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = gridDim.x, cta = blockIdx.x;
    const int T = p.T, k = p.k, E = p.E, d = p.d, f = p.f;
    const int NG = f / 16, NB = d / 64;
    const int npairs = T * k;
    const int nrt = (E + kWarps - 1) / kWarps;  // router CTA-tasks (8 rows each)
    const uint8_t *shrec = p.pool + int64_t(p.shared_slot) * p.slot_bytes;
    const uint32_t gu_codes = FMT == 2 ? uint32_t(d / 128) * 512u : uint32_t(d / 256) * 1536u;
    const uint32_t gu_scales = uint32_t(d / 128) * (FMT == 2 ? 128u : 64u);
    const uint32_t dn_codes = FMT == 2 ? uint32_t(f / 128) * 512u : uint32_t(f / 256) * 1536u;
    const uint32_t dn_scales = uint32_t(f / 128) * (FMT == 2 ? 128u : 64u);
    bool too_big = false;

    TRACE(0);
    // ------------------------------------------------------------ phase A
    if (tid == 0) {  // start the HBM reads of this CTA's phase-A task right away
        for (int task = cta; task < NG + nrt; task += G) {
            if (task < NG) {
                prefetch_l2(shrec + p.gate.codes_off + uint64_t(task) * gu_codes, gu_codes);
                prefetch_l2(shrec + p.up.codes_off + uint64_t(task) * gu_codes, gu_codes);
                prefetch_l2(shrec + p.gate.scales_off + uint64_t(task) * gu_scales, gu_scales);
                prefetch_l2(shrec + p.up.scales_off + uint64_t(task) * gu_scales, gu_scales);
            } else {
                const int e0 = kWarps * (task - NG);
                const int ne = min(kWarps, E - e0);
                prefetch_l2(p.Wr + size_t(e0) * d, uint32_t(ne) * uint32_t(d) * 4u);
            }
        }
    }
    // a router CTA-task (8 rows) loads its weights before anything else
    const int rtask = cta - NG;  // valid when 0 <= rtask < nrt (one phase-A task per CTA when G >= NG + nrt)
    const bool router_cta = G >= NG + nrt && rtask >= 0 && rtask < nrt;
    float4 wv[kRouterChunks];
    if (router_cta && kWarps * rtask + warp < E) router_load(p, kWarps * rtask + warp, lane, wv);
    {  // stage x and the slot table: every load of a thread is issued before any store
        constexpr int kXv = NT * kMaxDimDec / 8 / kThreads;  // uint4 per thread at most
        constexpr int kSv = kMaxEDec / kThreads;
        const uint4 *src = reinterpret_cast<const uint4 *>(p.x);
        uint4 *dst = reinterpret_cast<uint4 *>(sx);
        const int nx = T * d / 8;
        uint4 xv[kXv];
        int sv[kSv];
#pragma unroll
        for (int u = 0; u < kXv; ++u)
            if (tid + u * kThreads < nx) xv[u] = __ldg(src + tid + u * kThreads);
#pragma unroll
        for (int u = 0; u < kSv; ++u)
            if (tid + u * kThreads < E) sv[u] = __ldg(p.slot_of + tid + u * kThreads);
#pragma unroll
        for (int u = 0; u < kXv; ++u)
            if (tid + u * kThreads < nx) dst[tid + u * kThreads] = xv[u];
#pragma unroll
        for (int u = 0; u < kSv; ++u)
            if (tid + u * kThreads < E) s.slot[tid + u * kThreads] = sv[u];
        for (int i = cta * kThreads + tid; i < T * d; i += G * kThreads) p.y[i] = 0.f;
    }
    __syncthreads();
    TRACE(8);
    if (tid < kMaxTokDec) s.idx[0][tid] = tid;  // identity token list for the shared expert
    __syncthreads();
    bool xsum_ready = false;  // the router path does not need the block sums
    for (int task = cta; task < NG + nrt; task += G) {
        if (task < NG) {
            if (!xsum_ready) {
                stage_xsum(s, sx, NB, T, d);
                __syncthreads();
                xsum_ready = true;
            }
            gateup_task<FMT>(p, s, sx, shrec, task, T, s.idx[0], npairs);
            __syncthreads();
            if (tid == 0) {
                __threadfence();
                atomicAdd(p.done + kSharedIdx, 1u);
            }
        } else {
            const int e0 = kWarps * (task - NG);
            if (e0 + warp < E) {
                if (!router_cta) router_load(p, e0 + warp, lane, wv);
                router_row<NT>(p, sx, e0 + warp, lane, wv);
                if (warp == 0) TRACEW(10);
            }
            __syncthreads();
            if (tid == 0) {  // these router rows are written
                __threadfence();
                atomicAdd(p.ctr, unsigned(min(kWarps, E - e0)));
            }
        }
    }
    if (!xsum_ready) stage_xsum(s, sx, NB, T, d);  // for phase C (synchronised below)
    TRACE(1);
    // routing needs every logit: wait for all E router rows (not for the
    // shared expert's gate/up, which only phase D waits for)
    if (tid == 0) s.ok = wait_geq(p.ctr, unsigned(E), p.status);
    __syncthreads();
    if (!s.ok) goto finish;
    TRACE(2);

    // ------------------------------------------------------------ phase B
    if (warp < T) {
        // Top-k of token `warp` without selection rounds. A candidate is the
        // 64-bit (logit key << 32 | ~id): larger = larger logit, then lower id,
        // so the top k are the k largest candidates. The k-th largest lane
        // maximum L is a lower bound for the k-th largest candidate overall (the
        // k lanes whose maxima are >= L hold k candidates >= L), so only the
        // candidates >= L (usually a few more than k) are gathered and ranked.
        constexpr int M = kMaxEDec / 32;
        const float *row = p.logits + size_t(warp) * E;
        float lv[M];
#pragma unroll
        for (int m = 0; m < M; ++m) lv[m] = lane + 32 * m < E ? __ldcg(row + lane + 32 * m) : 0.f;
        if (warp == 0) {
            float sum_ = 0.f;
            for (int m = 0; m < M; ++m) sum_ += lv[m];
            if (sum_ == 12345.f) flag(p.status, 0);
            TRACEW(11);
        }
        uint64_t c[M];
        uint64_t mx = 0ull;
#pragma unroll
        for (int m = 0; m < M; ++m) {
            const int e = lane + 32 * m;
            c[m] = e < E ? (uint64_t(logit_key(lv[m])) << 32) | uint64_t(~uint32_t(e)) : 0ull;
            mx = c[m] > mx ? c[m] : mx;
        }
        int above = 0;  // lanes whose maximum beats ours
#pragma unroll
        for (int q = 0; q < 32; ++q) above += __shfl_sync(0xffffffffu, mx, q) > mx;
        const unsigned kth = __ballot_sync(0xffffffffu, above == k - 1);
        const uint64_t L = __shfl_sync(0xffffffffu, mx, __ffs(kth) - 1);
        int cnt = 0;
#pragma unroll
        for (int m = 0; m < M; ++m) cnt += c[m] >= L;
        int pre = cnt;  // inclusive prefix over lanes
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, pre, o);
            if (lane >= o) pre += v;
        }
        const int ncand = __shfl_sync(0xffffffffu, pre, 31);
        if (warp == 0) TRACEW(12);
        uint64_t *cand = s.cand[warp];
        int pos = pre - cnt;
#pragma unroll
        for (int m = 0; m < M; ++m)
            if (c[m] >= L) {
                if (pos < kCandMax) cand[pos] = c[m];
                ++pos;
            }
        __syncwarp();
        if (ncand <= 32) {  // one candidate per lane, ranked with shuffles
            const uint64_t me = lane < ncand ? cand[lane] : 0ull;
            int r = 0;
#pragma unroll
            for (int q = 0; q < 32; ++q) r += __shfl_sync(0xffffffffu, me, q) > me;
            if (lane < ncand && r < k) {
                const uint32_t key = uint32_t(me >> 32);
                const uint32_t u = (key & 0x80000000u) ? (key ^ 0x80000000u) : ~key;
                s.sel_v[warp][r] = __uint_as_float(u);
                s.sel_id[warp][r] = int(~uint32_t(me));
            }
        } else if (ncand <= kCandMax) {
            for (int i = lane; i < ncand; i += 32) {
                const uint64_t me = cand[i];
                int r = 0;
                for (int q = 0; q < ncand; ++q) r += cand[q] > me;
                if (r < k) {  // selected: keep its value and id (ordered by id below)
                    const uint32_t key = uint32_t(me >> 32);
                    const uint32_t u = (key & 0x80000000u) ? (key ^ 0x80000000u) : ~key;
                    s.sel_v[warp][r] = __uint_as_float(u);
                    s.sel_id[warp][r] = int(~uint32_t(me));
                }
            }
        } else {  // many near-equal maxima: k rounds of a warp-wide arg-max
            uint64_t best = 0ull;
#pragma unroll
            for (int m = 0; m < M; ++m) best = c[m] > best ? c[m] : best;
            for (int r = 0; r < k; ++r) {
                const uint32_t hk = uint32_t(best >> 32), hl = uint32_t(best);
                const uint32_t mk = __reduce_max_sync(0xffffffffu, hk);
                const uint32_t ml = __reduce_max_sync(0xffffffffu, hk == mk ? hl : 0u);
                if (lane == 0) {
                    const uint32_t u = (mk & 0x80000000u) ? (mk ^ 0x80000000u) : ~mk;
                    s.sel_v[warp][r] = __uint_as_float(u);
                    s.sel_id[warp][r] = int(~ml);
                }
                if (hk == mk && hl == ml) {
                    best = 0ull;
#pragma unroll
                    for (int m = 0; m < M; ++m) {
                        if (c[m] == ((uint64_t(mk) << 32) | ml)) c[m] = 0ull;
                        best = c[m] > best ? c[m] : best;
                    }
                }
            }
        }
    }
    if (warp < T) {
        __syncwarp();
        if (warp == 0) TRACEW(13);
        const int sel_id = lane < k ? s.sel_id[warp][lane] : 0;
        const float sel_v = lane < k ? s.sel_v[warp][lane] : 0.f;
        // sort the k selections by id and apply the softmax (normaliser summed in
        // ascending expert id, as moe_route does)
        const float vmax = __shfl_sync(0xffffffffu, sel_v, 0);
        const float ex = lane < k ? expf(sel_v - vmax) : 0.f;
        int rank = 0;
        for (int q = 0; q < k; ++q) rank += (__shfl_sync(0xffffffffu, sel_id, q) < sel_id);
        // ex of the a-th smallest id sits in the lane whose rank is a
        const unsigned rank_src = lane < k ? unsigned(rank) : 31u;
        float ex_by_id[kMaxK];
        int src_lane[kMaxK];
#pragma unroll
        for (int a = 0; a < kMaxK; ++a) {
            const unsigned hit = __ballot_sync(0xffffffffu, lane < k && rank_src == unsigned(a));
            src_lane[a] = hit ? __ffs(hit) - 1 : 0;
        }
#pragma unroll
        for (int a = 0; a < kMaxK; ++a) ex_by_id[a] = __shfl_sync(0xffffffffu, ex, src_lane[a]);
        float z = 0.f;
#pragma unroll
        for (int a = 0; a < kMaxK; ++a)
            if (a < k) z += ex_by_id[a];
        const float inv_z = 1.0f / z;
        if (lane < k) {
            s.idx[warp][rank] = sel_id;
            s.w[warp][rank] = ex * inv_z;
        }
    }
    __syncthreads();
    TRACE(6);
    if (T == 1 && tid < npairs) {  // one token: its list is already in id order
        s.pair_e[tid] = s.idx[0][tid];
        s.s_tok[tid] = 0;
        s.s_j[tid] = tid;
        s.inv[tid] = tid;
    } else if (tid < npairs) {  // stable sort of the pairs by (expert, pair index)
        const int pp = tid;
        const int e = s.idx[pp / k][pp % k];
        int rank = 0;
        for (int q = 0; q < npairs; ++q) {
            const int eq = s.idx[q / k][q % k];
            rank += (eq < e) || (eq == e && q < pp);
        }
        s.pair_e[rank] = e;
        s.s_tok[rank] = pp / k;
        s.s_j[rank] = pp % k;
        s.inv[pp] = rank;
    }
    __syncthreads();
    {  // experts with tokens, their segments, slots and miss bases (ballot scans)
        const bool in = tid < npairs;
        const bool first = in && (tid == 0 || s.pair_e[tid] != s.pair_e[tid - 1]);
        const unsigned fm = __ballot_sync(0xffffffffu, first);
        if (lane == 0 && warp < kMaxPairs / 32) s.first_mask[warp] = fm;
        __syncthreads();
        if (first) {
            int a = __popc(fm & ((1u << lane) - 1));
            for (int w = 0; w < warp; ++w) a += __popc(s.first_mask[w]);
            const int e = s.pair_e[tid];
            const int sl = s.slot[e];
            const bool bad = sl < -1 || sl >= p.num_slots;
            if (bad && cta == 0) flag(p.status, MOE_DEV_BAD_SLOT);
            s.act_e[a] = e;
            s.act_beg[a] = tid;
            s.act_slot[a] = bad ? -1 : sl;
        }
        if (tid == 0) {
            int na = 0;
            for (int w = 0; w < (npairs + 31) / 32; ++w) na += __popc(s.first_mask[w]);
            s.nact = na;
        }
        __syncthreads();
        const int na = s.nact;
        if (tid < na) s.act_cnt[tid] = (tid + 1 < na ? s.act_beg[tid + 1] : npairs) - s.act_beg[tid];
        __syncthreads();
        if (warp == 0) {  // resident list and miss bases over <= 128 actives, 32 at a time
            int nr = 0, nm = 0;
            for (int a0 = 0; a0 < na; a0 += 32) {
                const int a = a0 + lane;
                const bool act = a < na;
                const bool res = act && s.act_slot[a] >= 0;
                const int cm = act && !res ? s.act_cnt[a] : 0;
                const unsigned rm = __ballot_sync(0xffffffffu, res);
                int mpre = cm;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int v = __shfl_up_sync(0xffffffffu, mpre, o);
                    if (lane >= o) mpre += v;
                }
                if (act) s.act_mbase[a] = nm + mpre - cm;
                if (res) s.res[nr + __popc(rm & ((1u << lane) - 1))] = a;
                nr += __popc(rm);
                nm += __shfl_sync(0xffffffffu, mpre, 31);
            }
            if (lane == 0) {
                s.nres = nr;
                s.nmiss = nm;
            }
        }
    }
    __syncthreads();
    TRACE(5);
    {  // L2 prefetch of every selected expert, spread over the grid: the
        // concatenation of all resident experts' gate/up parts, then their down
        // parts and the shared expert's, is cut into G equal slices and the
        // threads of CTA c ask the L2 for the lines of slice c
        const int nres = s.nres;
        const uint32_t GU = uint32_t(p.down.codes_off);  // gate + up of one record
        const uint32_t DN = uint32_t(p.down.bytes);      // down of one record
        const uint32_t gu_all = uint32_t(nres) * GU;     // < 2^32: at most 128 records of < 8 MB
        const uint32_t total = gu_all + uint32_t(nres + 1) * DN;
        const uint32_t lo = uint32_t((uint64_t(total) * uint32_t(cta) / uint32_t(G))) & ~127u;
        const uint32_t hi = cta == G - 1 ? total : uint32_t((uint64_t(total) * uint32_t(cta + 1) / uint32_t(G))) & ~127u;
        // one 128-byte line per thread and step (GU and DN are multiples of 256)
        int r = -1;          // region of the current line and its start
        uint32_t r0 = 0, r1 = 0;
        const uint8_t *rsrc = nullptr;
        for (uint32_t o = lo + uint32_t(tid) * 128u; o < hi; o += uint32_t(kThreads) * 128u) {
            while (o >= r1) {  // advance to the region holding o (regions in order, each >= 1 step)
                ++r;
                r0 = r1;
                if (r < nres) {
                    r1 = r0 + GU;
                    rsrc = p.pool + int64_t(s.act_slot[s.res[r]]) * p.slot_bytes;
                } else {
                    const int q = r - nres;
                    r1 = r0 + DN;
                    const int slot = q < nres ? s.act_slot[s.res[q]] : p.shared_slot;
                    rsrc = p.pool + int64_t(slot) * p.slot_bytes + p.down.codes_off;
                }
            }
            asm volatile("prefetch.global.L2 [%0];" ::"l"(rsrc + (o - r0)));
        }
    }
    TRACE(3);
    // ------------------------------------------------------------ phase C
    {  // busy phase-A CTAs last; warp w handles K quads w, w+8, ... of every task,
        // and loads the next task's tiles before computing the current one
        const int ntasks = s.nres * NG;
        const int NQ = d / 256;
        const int g = lane >> 2, t = lane & 3;
        int task = G - 1 - cta;
        QuadRegs<FMT> ng, nu;  // tiles of the next task (quad = warp)
        auto load_task = [&](int tk, QuadRegs<FMT> &qg, QuadRegs<FMT> &qu) {
            const int ar = tk / NG, rg = tk % NG;
            const uint8_t *rec = p.pool + int64_t(s.act_slot[s.res[ar]]) * p.slot_bytes;
            quad_load<FMT>(rec, p.gate, rg, warp, lane, qg);
            quad_load<FMT>(rec, p.up, rg, warp, lane, qu);
        };
        const bool one_quad = NQ == kWarps;  // every warp owns exactly one quad
        if (one_quad && task < ntasks) load_task(task, ng, nu);
        uint32_t B1[4][8];     // one token: fragments of quad `warp`, built once
        float xs1[4][2];
        if (NT == 1 && one_quad) {
            build_b_bf16<FMT>(g == 0 ? sx : nullptr, warp, t, B1);
#pragma unroll
            for (int bq = 0; bq < 4; ++bq) {
                xs1[bq][0] = t == 0 ? s.xs[4 * warp + bq][0] : 0.f;
                xs1[bq][1] = 0.f;
            }
        }
        int nth = 0;
        for (; task < ntasks; task += G, ++nth) {
            const int ar = task / NG, rg = task % NG;
            const int a = s.res[ar];
            const int ntok = s.act_cnt[a];
            const int *tok = s.s_tok + s.act_beg[a];
            if (!one_quad) {  // general d: tiles loaded inside the task
                const uint8_t *rec = p.pool + int64_t(s.act_slot[a]) * p.slot_bytes;
                gateup_task<FMT>(p, s, sx, rec, rg, ntok, tok, s.act_beg[a]);
                __syncthreads();
                continue;
            }
            const QuadRegs<FMT> cg = ng, cu = nu;
            if (task + G < ntasks) load_task(task + G, ng, nu);
            float ag[4] = {0.f, 0.f, 0.f, 0.f}, au[4] = {0.f, 0.f, 0.f, 0.f};
            if (NT == 1) {
                quad_compute<FMT>(cg, B1, xs1, ag);
                quad_compute<FMT>(cu, B1, xs1, au);
            } else {
                const uint16_t *xrow = g < ntok ? sx + size_t(tok[g]) * d : nullptr;
                const int t0 = 2 * t < ntok ? tok[2 * t] : -1, t1 = 2 * t + 1 < ntok ? tok[2 * t + 1] : -1;
                uint32_t B[4][8];
                build_b_bf16<FMT>(xrow, warp, t, B);
                float xs[4][2];
#pragma unroll
                for (int bq = 0; bq < 4; ++bq) {
                    xs[bq][0] = t0 >= 0 ? s.xs[4 * warp + bq][t0] : 0.f;
                    xs[bq][1] = t1 >= 0 ? s.xs[4 * warp + bq][t1] : 0.f;
                }
                quad_compute<FMT>(cg, B, xs, ag);
                quad_compute<FMT>(cu, B, xs, au);
            }
            if (nth < 2 && warp == 0) TRACEW(nth == 0 ? 9 : 15);
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                s.red[warp][0][r][lane] = ag[r];
                s.red[warp][1][r][lane] = au[r];
            }
            __syncthreads();
            if (tid < 128) {
                const int L = tid >> 2, r = tid & 3;
                float A = 0.f, U = 0.f;
#pragma unroll
                for (int w = 0; w < kWarps; ++w) {
                    A += s.red[w][0][r][L];
                    U += s.red[w][1][r][L];
                }
                const int row = (L >> 2) + ((r & 2) ? 8 : 0);
                const int n = 2 * (L & 3) + (r & 1);
                if (n < ntok) p.h[size_t(s.act_beg[a] + n) * f + 16 * rg + row] = A / (1.0f + expf(-A)) * U;
            }
            __syncthreads();
            if (nth == 0) TRACE(14);
        }
    }
    // publish this CTA's h rows once (one fence), then count its tasks per expert
    if (tid == 0) {
        __threadfence();
        for (int task = G - 1 - cta; task < s.nres * NG; task += G) atomicAdd(p.done + task / NG, 1u);
    }

    TRACE(7);
    // ------------------------------------------------------------ phase D
    {
        const int nres = s.nres;
        const int nblk = d / 128;  // CTA-task = (expert, 8 row groups of d)
        const int NQf = f / 256;
        for (int task = cta; task < (nres + 1) * nblk; task += G) {
            const int ar = task / nblk, blk = task % nblk;
            const bool shared = ar == nres;
            const int a = shared ? 0 : s.res[ar];
            const int ntok = shared ? T : s.act_cnt[a];
            const int beg = shared ? npairs : s.act_beg[a];
            const int slot = shared ? p.shared_slot : s.act_slot[a];
            const uint8_t *rec = p.pool + int64_t(slot) * p.slot_bytes;
            const int rg = 8 * blk + warp;
            // this warp's first two weight tiles now (they do not depend on h)
            QuadRegs<FMT> q0, q1;
            quad_load<FMT>(rec, p.down, rg, 0, lane, q0);
            if (NQf > 1) quad_load<FMT>(rec, p.down, rg, 1, lane, q1);
            __syncthreads();  // previous task's readers of sh are done
            if (tid == 0) s.ok = wait_geq(p.done + (shared ? kSharedIdx : ar), unsigned(NG), p.status);
            __syncthreads();
            if (!s.ok) continue;
            {
                constexpr int kHv = NT * 1024 / 4 / kThreads + 1;  // float4 per thread at most
                const float4 *src = reinterpret_cast<const float4 *>(p.h + size_t(beg) * f);
                float4 *dst = reinterpret_cast<float4 *>(sh);
                const int nh = ntok * f / 4;
                float4 hv[kHv];
#pragma unroll
                for (int u = 0; u < kHv; ++u)
                    if (tid + u * kThreads < nh) hv[u] = __ldcg(src + tid + u * kThreads);
#pragma unroll
                for (int u = 0; u < kHv; ++u)
                    if (tid + u * kThreads < nh) dst[tid + u * kThreads] = hv[u];
            }
            __syncthreads();
            for (int job = warp; job < (f / 64) * ntok; job += kWarps) {  // block sums of h
                const int bb = job / ntok, n = job % ntok;
                const float2 v = *reinterpret_cast<const float2 *>(sh + size_t(n) * f + 64 * bb + 2 * lane);
                float sum = v.x + v.y;
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
                if (lane == 0) s.hsb[bb][n] = sum;
            }
            __syncthreads();
            const int g = lane >> 2, t = lane & 3;
            const float *hrow = g < ntok ? sh + size_t(g) * f : nullptr;
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
            for (int qd = 0; qd < NQf; ++qd) {  // tile qd computes while tile qd+2 loads
                QuadRegs<FMT> cur = q0;
                q0 = q1;
                if (qd + 2 < NQf) quad_load<FMT>(rec, p.down, rg, qd + 2, lane, q1);
                uint32_t B[4][8];
                build_b_f32_smem<FMT>(hrow, qd, t, B, too_big);
                float xs[4][2];
#pragma unroll
                for (int bq = 0; bq < 4; ++bq) {
                    xs[bq][0] = 2 * t < ntok ? s.hsb[4 * qd + bq][2 * t] : 0.f;
                    xs[bq][1] = 2 * t + 1 < ntok ? s.hsb[4 * qd + bq][2 * t + 1] : 0.f;
                }
                quad_compute<FMT>(cur, B, xs, acc);
            }
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int n = 2 * t + (r & 1);
                if (n < ntok) {
                    const int row = 16 * rg + g + ((r & 2) ? 8 : 0);
                    const int sp = beg + n;
                    const int tk = shared ? n : s.s_tok[sp];
                    const float gw = shared ? 1.f : s.w[tk][s.s_j[sp]];
                    atomicAdd(p.y + size_t(tk) * d + row, gw * acc[r]);
                }
            }
        }
    }

    // the last CTA publishes routing, permutation, slots and misses (nothing in
    // this launch reads them, so it happens after the compute)
    if (cta == G - 1) {
        for (int i = tid; i < npairs; i += kThreads) {
            const int t = i / k, j = i % k;
            if (p.topk_idx) p.topk_idx[i] = s.idx[t][j];
            if (p.topk_w) p.topk_w[i] = s.w[t][j];
            if (p.sorted_tok) p.sorted_tok[i] = s.s_tok[i];
            if (p.sorted_j) p.sorted_j[i] = s.s_j[i];
            if (p.inv) p.inv[i] = s.inv[i];
        }
        for (int e = tid; e <= E; e += kThreads) {
            int lo = 0, hi = s.nact;  // first active expert >= e
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if (s.act_e[mid] < e) lo = mid + 1; else hi = mid;
            }
            if (p.offsets) p.offsets[e] = lo < s.nact ? s.act_beg[lo] : npairs;
            if (p.counts && e < E) p.counts[e] = (lo < s.nact && s.act_e[lo] == e) ? s.act_cnt[lo] : 0;
        }
        if (p.active) {
            for (int a = tid; a < s.nact; a += kThreads) p.active[1 + a] = s.act_e[a];
            if (tid == 0) p.active[0] = s.nact;
        }
        for (int sp = tid; sp < npairs; sp += kThreads) {
            int a = 0;
            while (a + 1 < s.nact && s.act_beg[a + 1] <= sp) ++a;
            const bool res = s.act_slot[a] >= 0;
            const int pp = s.s_tok[sp] * k + s.s_j[sp];
            if (p.slot_of_pair) p.slot_of_pair[pp] = res ? s.act_slot[a] : -1;
            if (!res && p.miss) {
                const int mi = s.act_mbase[a] + (sp - s.act_beg[a]);
                if (mi < p.miss_cap) {
                    moe_miss m;
                    m.layer = p.layer;
                    m.expert = s.act_e[a];
                    m.token = s.s_tok[sp];
                    m.j = s.s_j[sp];
                    m.gate = s.w[m.token][m.j];
                    p.miss[mi] = m;
                }
            }
        }
        if (tid == 0) {
            if (p.miss_count) *p.miss_count = s.nmiss;
            if (s.nmiss > p.miss_cap && p.miss) flag(p.status, MOE_DEV_MISS_OVERFLOW);
        }
    }

finish:
    if (too_big) flag(p.status, MOE_DEV_NONFINITE);
    __syncthreads();
    TRACE(4);
    if (tid == 0) {
        __threadfence();
        s.last = atomicAdd(p.ctr + 1, 1u) == unsigned(G - 1);
    }
    __syncthreads();
    if (s.last) {  // every CTA is done with the counters: reset them for the next launch
        for (int i = tid; i <= kMaxPairs; i += kThreads) p.done[i] = 0u;
        if (tid == 0) p.ctr[0] = 0u;
        __threadfence();
        __syncthreads();
        if (tid == 0) {
            p.ctr[1] = 0u;
            __threadfence();
        }
    }
}

// Dynamic shared memory: T*d bf16 activations, then up to 8 rows of h (fp32).
constexpr size_t kDynSmemMax = size_t(kMaxTokDec) * kMaxDimDec * 2 + size_t(kMaxTokDec) * 1024 * 4;

size_t dyn_smem(int T, int d, int f) { return ((size_t(T) * d * 2 + 15) & ~size_t(15)) + size_t(T) * f * 4; }

struct LaunchCache {
    int grid[8][64] = {};
    bool ready[8][64] = {};
};
std::mutex g_mu;
LaunchCache g_cache;

template <int FMT, int NT>
moe_status launch(const DecodeParams &p, size_t smem, cudaStream_t stream) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    constexpr int ci = (FMT - 2) * 4 + (NT == 1 ? 0 : NT == 2 ? 1 : NT == 4 ? 2 : 3);
    int grid;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (!g_cache.ready[ci][dev]) {
            int sms = 0, per = 0;
            if (cudaFuncSetAttribute(decode_layer_kernel<FMT, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     int(kDynSmemMax)) != cudaSuccess ||
                cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
                cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, decode_layer_kernel<FMT, NT>, kThreads,
                                                              kDynSmemMax) != cudaSuccess ||
                per < 1) {
                cudaGetLastError();
                return MOE_ERR_CUDA;
            }
            g_cache.grid[ci][dev] = sms * std::min(per, kCtasPerSm);
            g_cache.ready[ci][dev] = true;
        }
        grid = g_cache.grid[ci][dev];
    }
    DecodeParams pp = p;
    void *args[] = {&pp};
    if (cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(decode_layer_kernel<FMT, NT>), dim3(grid),
                                    dim3(kThreads), args, smem, stream) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    return MOE_OK;
}

template <int FMT>
moe_status launch_fmt(const DecodeParams &p, size_t smem, cudaStream_t stream) {
    if (p.T <= 1) return launch<FMT, 1>(p, smem, stream);
    if (p.T <= 2) return launch<FMT, 2>(p, smem, stream);
    if (p.T <= 4) return launch<FMT, 4>(p, smem, stream);
    return launch<FMT, 8>(p, smem, stream);
}

size_t ws_align(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace
}  // namespace moe

using namespace moe;

MOE_API size_t moe_layer_decode_workspace_bytes(int T, int k, int f, int E) {
    if (T <= 0 || k <= 0 || f <= 0 || E <= 0) return 0;
    const size_t rows = size_t(T) * k + T;
    return ws_align(2 * sizeof(unsigned)) + ws_align((kMaxPairs + 1) * sizeof(unsigned)) +
           ws_align(size_t(T) * E * sizeof(float)) + ws_align(rows * f * sizeof(float));
}

MOE_API moe_status moe_layer_decode(const moe_qpool *W, const int32_t *slot_of, int32_t shared_slot, int32_t layer,
                                    const uint16_t *x, const float *Wr, const float *bias, int T, int d, int f, int E,
                                    int k, float *logits, int32_t *topk_idx, float *topk_w, int32_t *counts,
                                    int32_t *offsets, int32_t *sorted_tok, int32_t *sorted_j, int32_t *inv,
                                    int32_t *active, int32_t *slot_of_pair, moe_miss *miss, int32_t *miss_count,
                                    int32_t miss_cap, float *y, void *ws, size_t ws_bytes, int32_t *dev_status,
                                    moe_stream_t stream) {
    if (!W || T < 0 || E <= 0 || k <= 0 || miss_cap < 0) return MOE_ERR_INVALID_ARG;
    if (W->fmt != 2 && W->fmt != 3) return MOE_ERR_INVALID_ARG;
    if (W->d != d || W->f != f) return MOE_ERR_INVALID_ARG;
    if (!dims_ok(d, f) || d > kMaxDimDec || T > kMaxTokDec || E > kMaxEDec || k > kMaxK || k > E)
        return MOE_ERR_UNSUPPORTED;
    if (T == 0) return MOE_OK;
    if (!slot_of || !x || !Wr || !y) return MOE_ERR_INVALID_ARG;
    if (miss_cap > 0 && !miss) return MOE_ERR_INVALID_ARG;
    const ExpertGeom eg = expert_geom(W->fmt, d, f);
    if (!W->base || W->num_slots <= 0 || W->slot_bytes < int64_t(eg.bytes) || W->slot_bytes % 256 ||
        reinterpret_cast<uintptr_t>(W->base) % 256 || shared_slot < 0 || shared_slot >= W->num_slots)
        return MOE_ERR_INVALID_ARG;
    if (!ws || ws_bytes < moe_layer_decode_workspace_bytes(T, k, f, E)) return MOE_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(ws) % 256) return MOE_ERR_INVALID_ARG;
    DecodeParams p;
    p.pool = static_cast<const uint8_t *>(W->base);
    p.slot_bytes = W->slot_bytes;
    p.num_slots = W->num_slots;
    p.slot_of = slot_of;
    p.shared_slot = shared_slot;
    p.layer = layer;
    p.x = x;
    p.Wr = Wr;
    p.bias = bias;
    p.T = T;
    p.d = d;
    p.f = f;
    p.E = E;
    p.k = k;
    p.topk_idx = topk_idx;
    p.topk_w = topk_w;
    p.counts = counts;
    p.offsets = offsets;
    p.sorted_tok = sorted_tok;
    p.sorted_j = sorted_j;
    p.inv = inv;
    p.active = active;
    p.slot_of_pair = slot_of_pair;
    p.miss = miss;
    p.miss_count = miss_count;
    p.miss_cap = miss_cap;
    p.y = y;
    p.status = dev_status;
    unsigned char *w = static_cast<unsigned char *>(ws);
    p.ctr = reinterpret_cast<unsigned *>(w);
    w += ws_align(2 * sizeof(unsigned));
    p.done = reinterpret_cast<unsigned *>(w);
    w += ws_align((kMaxPairs + 1) * sizeof(unsigned));
    float *lg = reinterpret_cast<float *>(w);
    w += ws_align(size_t(T) * E * sizeof(float));
    p.logits = logits ? logits : lg;
    p.h = reinterpret_cast<float *>(w);
    p.gate = eg.m[0];
    p.up = eg.m[1];
    p.down = eg.m[2];
    if (dyn_smem(T, d, f) > kDynSmemMax) return MOE_ERR_UNSUPPORTED;
    const size_t smem = dyn_smem(T, d, f);
    return W->fmt == 2 ? launch_fmt<2>(p, smem, as_cuda(stream)) : launch_fmt<3>(p, smem, as_cuda(stream));
}

#ifdef MOE_DECODE_TRACE
// Trace builds only: copy the phase timestamps to host memory.
MOE_API int moe_decode_trace_read(void *dst) {  // 4096 CTAs x (16 timestamps, 16 clocks)
    return int(cudaMemcpyFromSymbol(dst, moe_decode_trace, sizeof(moe_decode_trace)));
}
#endif
