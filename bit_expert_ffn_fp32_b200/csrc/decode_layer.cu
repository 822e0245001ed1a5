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
        }                                                                                             \
    } while (0)
#define TRACEW(i)                                                                                     \
    do {                                                                                              \
        if ((threadIdx.x & 31) == 0) {                                                                \
            unsigned long long t_;                                                                    \
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                                    \
            moe_decode_trace[blockIdx.x * 32 + (i)] = t_;                                             \
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
constexpr unsigned long long kWaitSteps = 1ull << 27;  // polls: >= 4 s of 32 ns sleeps
constexpr int kMaxSlots = 8;  // weight-ring slots at most
constexpr int kMaxFDec = 1024;  // expert width f (h staging and B fragments)
constexpr int kCBatch = 4;      // gate/up units computed in one pass (one token)
static_assert(kCBatch * kWarps * 2 * 16 <= kWarps * 2 * 4 * 32, "batched partials fit in red[]");
static_assert(kMaxSlots <= kWarps, "one warp announces each initial ring unit");

// Dynamic shared memory: T*d bf16 activations, T rows of h (fp32), then the
// weight ring from this 128-byte aligned offset.
__host__ __device__ inline size_t ring_off(int T, int d, int f) {
    return ((((size_t(T) * d * 2 + 15) & ~size_t(15)) + size_t(T) * f * 4) + 127) & ~size_t(127);
}

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
    // shared-memory weight ring of phases C and D: nslots slots of rslot bytes;
    // per row group, the codes and scales bytes of gate/up (gu_*) and down (dn_*)
    int nslots;
    uint32_t rslot, gu_cb, gu_sb, dn_cb, dn_sb;
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
    float hsb[kMaxFDec / 64][kMaxTokDec];   // block sums of the staged h rows
    uint64_t cand[kMaxTokDec][kCandMax];    // top-k candidates per token
    float sel_v[kMaxTokDec][kMaxK];
    int sel_id[kMaxTokDec][kMaxK];
    unsigned first_mask[kMaxPairs / 32];    // pair s starts a new expert
    uint64_t full[kMaxSlots];               // weight ring: slot filled (bulk-copy bytes landed)
    // B fragments of the staged h rows, built once per down unit and shared by
    // every warp: quad qd, fragment registers 4*r4..4*r4+3, lane: [qd][r4][lane]
    uint4 bfrag[kMaxFDec / 256][8][32];
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
    // the iteration cap ends the wait even if the timer stood still (each step sleeps >= 32 ns)
    for (unsigned long long it = 0; ld_acquire(p) < target; ++it) {
        if (globaltimer() - t0 > kWaitNs || it > kWaitSteps) {
            flag(status, MOE_DEV_TIMEOUT);
            return false;
        }
        __nanosleep(32);
    }
    return true;
}

// Weight ring: bulk copies global -> this CTA's shared memory that complete
// on an mbarrier (transaction bytes), and a bounded wait for a slot's phase.
__device__ __forceinline__ uint32_t saddr(const void *p) { return uint32_t(__cvta_generic_to_shared(p)); }
__device__ __forceinline__ void ring_expect(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(saddr(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void ring_copy(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     saddr(dst)),
                 "l"(src), "r"(bytes), "r"(saddr(bar))
                 : "memory");
}
__device__ __forceinline__ bool ring_test(uint64_t *bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n.reg .pred q;\nmbarrier.try_wait.parity.shared::cta.b64 q, [%1], %2;\nselp.u32 %0, 1, 0, q;\n}"
        : "=r"(done)
        : "r"(saddr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}
// false after kWaitNs, or kWaitSteps polls (the caller flags MOE_DEV_TIMEOUT)
__device__ bool ring_wait(uint64_t *bar, uint32_t parity) {
    if (ring_test(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    for (unsigned long long it = 0; !ring_test(bar, parity); ++it) {
        if (globaltimer() - t0 > kWaitNs || it > kWaitSteps) return false;
        if (it > 1024) __nanosleep(32);
    }
    return true;
}

// One CTA runs the two waits above against objects nothing completes (a device
// counter below target, a fresh mbarrier phase with no arrival): both give up
// with MOE_DEV_TIMEOUT; elapsed[0..1] receive their durations.
__global__ void wait_probe_kernel(const unsigned *counter, unsigned target, unsigned long long *elapsed,
                                  int32_t *status) {
    __shared__ uint64_t bar;
    if (threadIdx.x != 0) return;
    const unsigned long long t0 = globaltimer();
    wait_geq(counter, target, status);
    const unsigned long long t1 = globaltimer();
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(saddr(&bar)) : "memory");
    if (!ring_wait(&bar, 0u)) flag(status, MOE_DEV_TIMEOUT);
    elapsed[0] = t1 - t0;
    elapsed[1] = globaltimer() - t1;
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

// Packed codes and scales of one 16-row x 256-column tile (columns 256qd..)
// from a row group's bytes in shared memory, laid out as in the record: codes
// at cb, scales at sb (the offsets of q2_chunk_off / q3_word_off / scale_off
// relative to the row group's start).
template <int FMT>
__device__ __forceinline__ void quad_load_smem(const uint8_t *cb, const uint8_t *sb, int qd, int lane,
                                               QuadRegs<FMT> &q) {
    const int g = lane >> 2;
    if constexpr (FMT == 2) {
        q.c0 = *reinterpret_cast<const uint4 *>(cb + ((2 * qd) * 32 + lane) * 16);
        q.c1 = *reinterpret_cast<const uint4 *>(cb + ((2 * qd + 1) * 32 + lane) * 16);
        q.s0 = *reinterpret_cast<const uint4 *>(sb + ((2 * qd) * 8 + g) * 16);
        q.s1 = *reinterpret_cast<const uint4 *>(sb + ((2 * qd + 1) * 8 + g) * 16);
    } else {
#pragma unroll
        for (int w = 0; w < 3; ++w) {
            const uint4 v = *reinterpret_cast<const uint4 *>(cb + qd * 1536 + w * 512 + lane * 16);
            q.W[4 * w + 0] = v.x;
            q.W[4 * w + 1] = v.y;
            q.W[4 * w + 2] = v.z;
            q.W[4 * w + 3] = v.w;
        }
        q.s0 = *reinterpret_cast<const uint2 *>(sb + ((2 * qd) * 8 + g) * 8);
        q.s1 = *reinterpret_cast<const uint2 *>(sb + ((2 * qd + 1) * 8 + g) * 8);
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
    float *sh = reinterpret_cast<float *>(dyn + ((size_t(p.T) * p.d * 2 + 15) & ~size_t(15)));  // [T][f] h
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = gridDim.x, cta = blockIdx.x;
    const int T = p.T, k = p.k, E = p.E, d = p.d, f = p.f;
    const int NG = f / 16, NB = d / 64;
    const int npairs = T * k;
    const int nrt = (E + kWarps - 1) / kWarps;  // router CTA-tasks (8 rows each)
    const uint8_t *shrec = p.pool + int64_t(p.shared_slot) * p.slot_bytes;
    const uint32_t gu_codes = FMT == 2 ? uint32_t(d / 128) * 512u : uint32_t(d / 256) * 1536u;
    const uint32_t gu_scales = uint32_t(d / 128) * (FMT == 2 ? 128u : 64u);
    bool too_big = false;
    int ring_issued = 0, ring_used = 0;  // thread 0: weight-ring units copied / consumed

    TRACE(0);
    if (tid == 0) {
        for (int i = 0; i < kMaxSlots; ++i)
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(saddr(&s.full[i])) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
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
    if (T == 1) {
        if (warp == 0) {  // one token: its k experts (id order) are the active experts, one pair each
            const bool in = lane < k;
            int sl = -1;
            if (in) {
                const int e = s.idx[0][lane];
                s.pair_e[lane] = e;
                s.s_tok[lane] = 0;
                s.s_j[lane] = lane;
                s.inv[lane] = lane;
                sl = s.slot[e];
                const bool bad = sl < -1 || sl >= p.num_slots;
                if (bad && cta == 0) flag(p.status, MOE_DEV_BAD_SLOT);
                if (bad) sl = -1;
                s.act_e[lane] = e;
                s.act_beg[lane] = lane;
                s.act_cnt[lane] = 1;
                s.act_slot[lane] = sl;
            }
            const unsigned rm = __ballot_sync(0xffffffffu, in && sl >= 0);
            const unsigned mm = __ballot_sync(0xffffffffu, in && sl < 0);
            const unsigned lt = (1u << lane) - 1u;
            if (in) s.act_mbase[lane] = __popc(mm & lt);
            if (in && sl >= 0) s.res[__popc(rm & lt)] = lane;
            if (lane == 0) {
                s.nact = k;
                s.nres = __popc(rm);
                s.nmiss = __popc(mm);
            }
        }
    } else {
        if (tid < npairs) {  // stable sort of the pairs by (expert, pair index)
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
    }
    __syncthreads();
    TRACE(5);
    {
        // ------------------------------------------------------------ weight ring
        // This CTA's units: its gate/up tasks (task = G-1-cta + u*G < nres*NG,
        // busy phase-A CTAs last), then its down tasks (a contiguous range of
        // tasks < (nres+1)*nblk; a down task is an expert x 8 row groups of d,
        // the shared expert last). Thread 0 bulk-copies a unit's packed bytes
        // (contiguous per row group in the record) into ring slot u % NS as soon
        // as the routing tables exist, the first NS units at once, and refills a
        // slot with unit u + NS once unit u has been computed.
        const int NQ = d / 256, NQf = f / 256, nblk = d / 128;
        const int nres = s.nres;
        const int ctasks = nres * NG, dtasks = (nres + 1) * nblk;
        const int cfirst = G - 1 - cta;
        const int nC = ctasks > cfirst ? (ctasks - cfirst + G - 1) / G : 0;
        // down tasks: a contiguous range per CTA (consecutive tasks mostly share an
        // expert, whose staged h and B fragments are then reused)
        const int dlo = int(int64_t(dtasks) * cta / G), nD = int(int64_t(dtasks) * (cta + 1) / G) - dlo;
        const int nU = nC + nD, NS = p.nslots;
        uint8_t *ring = dyn + ring_off(T, d, f);
        // copy c (0..3 gate/up: gate codes, gate scales, up codes, up scales;
        // 0..1 down: codes, scales) of unit u; one thread per copy
        auto issue_copy = [&](int u, int c) {
            uint8_t *dst = ring + size_t(u % NS) * p.rslot;
            uint64_t *bar = &s.full[u % NS];
            if (u < nC) {
                const int task = cfirst + u * G, ar = task / NG, rg = task % NG;
                const uint8_t *rec = p.pool + int64_t(s.act_slot[s.res[ar]]) * p.slot_bytes;
                const MatGeom &m = c < 2 ? p.gate : p.up;
                const uint32_t off = (c >> 1) * (p.gu_cb + p.gu_sb) + (c & 1) * p.gu_cb;
                if (c & 1)
                    ring_copy(dst + off, rec + m.scales_off + uint64_t(rg) * p.gu_sb, p.gu_sb, bar);
                else
                    ring_copy(dst + off, rec + m.codes_off + uint64_t(rg) * p.gu_cb, p.gu_cb, bar);
            } else if (c < 2) {
                const int task = dlo + (u - nC), ar = task / nblk, blk = task % nblk;
                const int slot = ar == nres ? p.shared_slot : s.act_slot[s.res[ar]];
                const uint8_t *rec = p.pool + int64_t(slot) * p.slot_bytes;
                if (c)
                    ring_copy(dst + 8 * p.dn_cb, rec + p.down.scales_off + uint64_t(8 * blk) * p.dn_sb,
                              8u * p.dn_sb, bar);
                else
                    ring_copy(dst, rec + p.down.codes_off + uint64_t(8 * blk) * p.dn_cb, 8u * p.dn_cb, bar);
            }
        };
        auto unit_bytes = [&](int u) { return u < nC ? 2u * (p.gu_cb + p.gu_sb) : 8u * (p.dn_cb + p.dn_sb); };
        auto issue = [&](int u) {  // one thread, all copies of unit u
            ring_expect(&s.full[u % NS], unit_bytes(u));
            for (int c = 0; c < 4; ++c) issue_copy(u, c);
        };
        {  // the first min(nU, NS) units at once: warp u announces unit u, its lanes 0..3 copy
            const int n0 = min(nU, NS);
            if (warp < n0) {
                if (lane == 0) ring_expect(&s.full[warp], unit_bytes(warp));
                __syncwarp();
                if (lane < 4) issue_copy(warp, lane);
            }
            ring_issued = n0;  // meaningful in thread 0
        }
        TRACE(3);
        // every thread waits for unit u's bytes itself; false (all threads) on timeout
        auto await_unit = [&](int u) -> bool {
            const bool got = ring_wait(&s.full[u % NS], uint32_t(u / NS) & 1u);
            if (!got && tid == 0) flag(p.status, MOE_DEV_TIMEOUT);
            const bool all = __syncthreads_and(got) != 0;
            if (all && tid == 0) ++ring_used;
            return all;
        };

        // ------------------------------------------------------------ phase C
        const int g = lane >> 2, t = lane & 3;
        const bool one_quad = NQ == kWarps;  // every warp owns exactly one quad
        uint32_t B1[4][8];                   // one token: fragments of quad `warp`, built once
        float xs1[4][2];
        if (NT == 1 && one_quad) {
            build_b_bf16<FMT>(g == 0 ? sx : nullptr, warp, t, B1);
#pragma unroll
            for (int bq = 0; bq < 4; ++bq) {
                xs1[bq][0] = t == 0 ? s.xs[4 * warp + bq][0] : 0.f;
                xs1[bq][1] = 0.f;
            }
        }
        // One token and all of this CTA's gate/up units in the ring at once: wait
        // for all of them, compute every unit's quad `warp` back to back (their
        // MMA chains interleave), then one reduction over warps for all units
        // (same summation order as the per-unit path below).
        const bool batch = NT == 1 && one_quad && nC <= min(NS, kCBatch);
        if (batch) {
            // every thread waits for each unit itself and computes it at once:
            // no barrier until all units are done
            bool got = true;
            float ag[kCBatch][4], au[kCBatch][4];
#pragma unroll
            for (int i = 0; i < kCBatch; ++i) {
                if (i < nC) {
                    got = got && ring_wait(&s.full[i], 0u);
                    if (i == 0) TRACE(16);
                    const uint8_t *slot = ring + size_t(i) * p.rslot;
                    QuadRegs<FMT> qg, qu;
                    quad_load_smem<FMT>(slot, slot + p.gu_cb, warp, lane, qg);
                    quad_load_smem<FMT>(slot + p.gu_cb + p.gu_sb, slot + 2 * p.gu_cb + p.gu_sb, warp, lane, qu);
#pragma unroll
                    for (int r = 0; r < 4; ++r) ag[i][r] = au[i][r] = 0.f;
                    quad_compute<FMT>(qg, B1, xs1, ag[i]);
                    quad_compute<FMT>(qu, B1, xs1, au[i]);
                }
            }
            if (warp == 0) TRACEW(9);
            if (!got && tid == 0) flag(p.status, MOE_DEV_TIMEOUT);
            if (!__syncthreads_and(got)) goto finish;
            if (tid == 0) ring_used = nC;
            // token 0 sits in lanes t == 0: rows g (r = 0) and g + 8 (r = 2)
            float(*red1)[kWarps][2][16] = reinterpret_cast<float(*)[kWarps][2][16]>(&s.red[0][0][0][0]);
            if (t == 0) {
#pragma unroll
                for (int i = 0; i < kCBatch; ++i) {
                    if (i < nC) {
                        red1[i][warp][0][g] = ag[i][0];
                        red1[i][warp][0][g + 8] = ag[i][2];
                        red1[i][warp][1][g] = au[i][0];
                        red1[i][warp][1][g + 8] = au[i][2];
                    }
                }
            }
            __syncthreads();
            TRACE(17);
            if (tid < nC * 16) {
                const int i = tid >> 4, row = tid & 15;
                const int task = cfirst + i * G, ar = task / NG, rg = task % NG;
                float A = 0.f, U = 0.f;
#pragma unroll
                for (int w = 0; w < kWarps; ++w) {
                    A += red1[i][w][0][row];
                    U += red1[i][w][1][row];
                }
                p.h[size_t(s.act_beg[s.res[ar]]) * f + 16 * rg + row] = A / (1.0f + expf(-A)) * U;
            }
            __syncthreads();  // slots and red[] read by everyone
            if (tid == 0)
                while (ring_issued < nU && ring_issued < nC + NS) issue(ring_issued++);
            TRACE(14);
        }
        for (int u = 0; !batch && u < nC; ++u) {
            const int task = cfirst + u * G, ar = task / NG, rg = task % NG;
            const int a = s.res[ar];
            const int ntok = s.act_cnt[a];
            const int *tok = s.s_tok + s.act_beg[a];
            if (!await_unit(u)) goto finish;
            if (u == 0) TRACE(16);
            const uint8_t *slot = ring + size_t(u % NS) * p.rslot;
            float ag[4] = {0.f, 0.f, 0.f, 0.f}, au[4] = {0.f, 0.f, 0.f, 0.f};
            for (int qd = warp; qd < NQ; qd += kWarps) {
                QuadRegs<FMT> qg, qu;
                quad_load_smem<FMT>(slot, slot + p.gu_cb, qd, lane, qg);
                quad_load_smem<FMT>(slot + p.gu_cb + p.gu_sb, slot + 2 * p.gu_cb + p.gu_sb, qd, lane, qu);
                if (NT == 1 && one_quad) {
                    quad_compute<FMT>(qg, B1, xs1, ag);
                    quad_compute<FMT>(qu, B1, xs1, au);
                } else {
                    const uint16_t *xrow = g < ntok ? sx + size_t(tok[g]) * d : nullptr;
                    const int t0 = 2 * t < ntok ? tok[2 * t] : -1, t1 = 2 * t + 1 < ntok ? tok[2 * t + 1] : -1;
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
            }
            if (u < 2 && warp == 0) TRACEW(u == 0 ? 9 : 15);
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                s.red[warp][0][r][lane] = ag[r];
                s.red[warp][1][r][lane] = au[r];
            }
            __syncthreads();
            if (u == 0) TRACE(17);
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
            __syncthreads();  // slot and red[] read by everyone
            if (tid == 0 && ring_issued < nU) issue(ring_issued++);
            if (u == 0) TRACE(14);
        }
        // publish this CTA's h rows (written before the last barrier): one fence
        // and one count per task, by as many threads
        for (int u = tid; u < nC; u += kThreads) {
            __threadfence();
            atomicAdd(p.done + (cfirst + u * G) / NG, 1u);
        }

        TRACE(7);
        // ------------------------------------------------------------ phase D
        int staged = -1;  // expert whose h, block sums and B fragments are in shared memory
        for (int u = nC; u < nU; ++u) {
            const int task = dlo + (u - nC), ar = task / nblk, blk = task % nblk;
            const bool shared = ar == nres;
            const int a = shared ? 0 : s.res[ar];
            const int ntok = shared ? T : s.act_cnt[a];
            const int beg = shared ? npairs : s.act_beg[a];
            const int rg = 8 * blk + warp;
            if (!await_unit(u)) goto finish;
            if (u == nC) TRACE(18);
            if (ar != staged) {  // the expert's first unit here: wait for its h, stage it
                staged = ar;
                if (tid == 0) s.ok = wait_geq(p.done + (shared ? kSharedIdx : ar), unsigned(NG), p.status);
                __syncthreads();
                if (!s.ok) goto finish;
                if (u == nC) TRACE(19);
                {  // the expert's h rows (written by other CTAs: read through L2) into shared memory
                    constexpr int kHv = NT * kMaxFDec / 4 / kThreads + 1;  // float4 per thread at most
                    const float4 *src = reinterpret_cast<const float4 *>(p.h + size_t(beg) * f);
                    float4 *dst = reinterpret_cast<float4 *>(sh);
                    const int nh = ntok * f / 4;
                    float4 hv[kHv];
    #pragma unroll
                    for (int v = 0; v < kHv; ++v)
                        if (tid + v * kThreads < nh) hv[v] = __ldcg(src + tid + v * kThreads);
    #pragma unroll
                    for (int v = 0; v < kHv; ++v)
                        if (tid + v * kThreads < nh) dst[tid + v * kThreads] = hv[v];
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
                // B fragments of every quad of h (element (k, n=gg) of slot rho of
                // block bq for lane (gg, tt): columns 256qd + 64bq + slot_k(rho, tt),
                // divided by 2^slot_exp), one 16-byte entry per thread and step
                for (int e = tid; e < NQf * 256; e += kThreads) {
                    const int qd = e >> 8, ln = (e >> 3) & 31, r4 = e & 7;
                    const int gg = ln >> 2, tt = ln & 3, bq = r4 >> 1;
                    const float *src = gg < ntok ? sh + size_t(gg) * f + 256 * qd + 64 * bq : nullptr;
                    uint32_t v[4];
    #pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int rho = (r4 & 1) * 4 + j;
                        float lo = 0.f, hi = 0.f;
                        if (src) {
                            const float2 hv = *reinterpret_cast<const float2 *>(src + slot_k(rho, tt, 0));
                            lo = hv.x;
                            hi = hv.y;
                            too_big |= !(fabsf(lo) <= 65504.f) || !(fabsf(hi) <= 65504.f);
                        }
                        const float sc = __int_as_float((127 - slot_exp<FMT>(bq, rho)) << 23);  // 2^-exp
                        v[j] = pack_half2(lo * sc, hi * sc);
                    }
                    s.bfrag[qd][r4][ln] = make_uint4(v[0], v[1], v[2], v[3]);
                }
                __syncthreads();
            }
            if (u == nC) TRACE(20);
            const uint8_t *slot = ring + size_t(u % NS) * p.rslot;
            const uint8_t *cb = slot + warp * p.dn_cb, *sb = slot + 8 * p.dn_cb + warp * p.dn_sb;
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
            for (int qd = 0; qd < NQf; ++qd) {
                QuadRegs<FMT> q;
                quad_load_smem<FMT>(cb, sb, qd, lane, q);
                uint32_t B[4][8];
#pragma unroll
                for (int r4 = 0; r4 < 8; ++r4) {
                    const uint4 v = s.bfrag[qd][r4][lane];
                    B[r4 >> 1][(r4 & 1) * 4 + 0] = v.x;
                    B[r4 >> 1][(r4 & 1) * 4 + 1] = v.y;
                    B[r4 >> 1][(r4 & 1) * 4 + 2] = v.z;
                    B[r4 >> 1][(r4 & 1) * 4 + 3] = v.w;
                }
                float xs[4][2];
#pragma unroll
                for (int bq = 0; bq < 4; ++bq) {
                    xs[bq][0] = 2 * t < ntok ? s.hsb[4 * qd + bq][2 * t] : 0.f;
                    xs[bq][1] = 2 * t + 1 < ntok ? s.hsb[4 * qd + bq][2 * t + 1] : 0.f;
                }
                quad_compute<FMT>(q, B, xs, acc);
            }
            if (u == nC && warp == 0) TRACEW(21);
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
            __syncthreads();  // slot, sh, bfrag and hsb read by everyone
            if (u == nC) TRACE(22);
            if (tid == 0 && ring_issued < nU) issue(ring_issued++);
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
    if (tid == 0)  // copies still in flight (error paths only) land before the CTA leaves
        for (int u = ring_used; u < ring_issued; ++u)
            if (!ring_wait(&s.full[u % p.nslots], uint32_t(u / p.nslots) & 1u)) break;
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

struct LaunchCache {
    int grid[8][64] = {};
    int avail[8][64] = {};  // dynamic shared memory a CTA can have
    bool ready[8][64] = {};
};
std::mutex g_mu;
LaunchCache g_cache;

template <int FMT, int NT>
moe_status launch(DecodeParams p, cudaStream_t stream) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    constexpr int ci = (FMT - 2) * 4 + (NT == 1 ? 0 : NT == 2 ? 1 : NT == 4 ? 2 : 3);
    int grid, avail;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (!g_cache.ready[ci][dev]) {
            int sms = 0, per = 0, optin = 0;
            cudaFuncAttributes fa;
            if (cudaFuncGetAttributes(&fa, decode_layer_kernel<FMT, NT>) != cudaSuccess ||
                cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
                cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
                cudaGetLastError();
                return MOE_ERR_CUDA;
            }
            const int av = optin - int(fa.sharedSizeBytes);
            if (av <= 0 ||
                cudaFuncSetAttribute(decode_layer_kernel<FMT, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, av) !=
                    cudaSuccess ||
                cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, decode_layer_kernel<FMT, NT>, kThreads, av) !=
                    cudaSuccess ||
                per < 1) {
                cudaGetLastError();
                return MOE_ERR_CUDA;
            }
            g_cache.grid[ci][dev] = sms * std::min(per, kCtasPerSm);
            g_cache.avail[ci][dev] = av;
            g_cache.ready[ci][dev] = true;
        }
        grid = g_cache.grid[ci][dev];
        avail = g_cache.avail[ci][dev];
    }
    const size_t base = ring_off(p.T, p.d, p.f);
    if (size_t(avail) < base + 2 * size_t(p.rslot)) return MOE_ERR_UNSUPPORTED;
    p.nslots = int(std::min<size_t>(kMaxSlots, (size_t(avail) - base) / p.rslot));
    const size_t smem = base + size_t(p.nslots) * p.rslot;
    void *args[] = {&p};
    if (cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(decode_layer_kernel<FMT, NT>), dim3(grid),
                                    dim3(kThreads), args, smem, stream) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    return MOE_OK;
}

template <int FMT>
moe_status launch_fmt(const DecodeParams &p, cudaStream_t stream) {
    if (p.T <= 1) return launch<FMT, 1>(p, stream);
    if (p.T <= 2) return launch<FMT, 2>(p, stream);
    if (p.T <= 4) return launch<FMT, 4>(p, stream);
    return launch<FMT, 8>(p, stream);
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
    if (!dims_ok(d, f) || d > kMaxDimDec || f > kMaxFDec || T > kMaxTokDec || E > kMaxEDec || k > kMaxK || k > E)
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
    // bytes of one row group's codes and scales (contiguous in the record), and
    // the ring slot: a gate/up task (both matrices) or a down task (8 row groups)
    const int fmt = W->fmt;
    auto cbytes = [&](const MatGeom &m) {
        return uint32_t(fmt == 2 ? q2_chunk_off(m, 1, 0, 0) - q2_chunk_off(m, 0, 0, 0)
                                 : q3_word_off(m, 1, 0, 0, 0) - q3_word_off(m, 0, 0, 0, 0));
    };
    auto sbytes = [&](const MatGeom &m) { return uint32_t(scale_off(m, fmt, 1, 0, 0) - scale_off(m, fmt, 0, 0, 0)); };
    p.gu_cb = cbytes(p.gate);
    p.gu_sb = sbytes(p.gate);
    p.dn_cb = cbytes(p.down);
    p.dn_sb = sbytes(p.down);
    if ((p.gu_cb | p.gu_sb | p.dn_cb | p.dn_sb) % 16 ||
        (p.gate.codes_off | p.gate.scales_off | p.up.codes_off | p.up.scales_off | p.down.codes_off |
         p.down.scales_off) % 16 ||
        cbytes(p.up) != p.gu_cb || sbytes(p.up) != p.gu_sb)
        return MOE_ERR_UNSUPPORTED;
    p.rslot = (std::max(2u * (p.gu_cb + p.gu_sb), 8u * (p.dn_cb + p.dn_sb)) + 127u) & ~127u;
    p.nslots = 0;
    return fmt == 2 ? launch_fmt<2>(p, as_cuda(stream)) : launch_fmt<3>(p, as_cuda(stream));
}

MOE_API moe_status moe_debug_wait_probe(const uint32_t *counter, uint32_t target, uint64_t *elapsed_ns,
                                        int32_t *dev_status, moe_stream_t stream) {
    if (!counter || !elapsed_ns || !dev_status) return MOE_ERR_INVALID_ARG;
    wait_probe_kernel<<<1, 32, 0, as_cuda(stream)>>>(counter, target,
                                                     reinterpret_cast<unsigned long long *>(elapsed_ns), dev_status);
    return launch_status();
}

#ifdef MOE_DECODE_TRACE
// Trace builds only: copy the phase timestamps to host memory.
MOE_API int moe_decode_trace_read(void *dst) {  // 4096 CTAs x 32 timestamps
    return int(cudaMemcpyFromSymbol(dst, moe_decode_trace, sizeof(moe_decode_trace)));
}
#endif
