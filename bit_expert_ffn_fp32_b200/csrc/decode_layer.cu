// Whole MoE layers for a few tokens (decode, MTP verify) in one cooperative
// launch of thread-block clusters: one layer (moe_layer_decode) or a stack of
// layers (moe_stack_decode).
//
// Per token the router scores the layer's experts, the top k (10 of 512 in
// "个人开发者用 AI 十天写出 Strata 引擎，让 12GB 显存跑起 1250 亿参数的 Qwen 3.8 Flash
// Next", section "1250 亿参数，每个词只用得上 2%") run as SwiGLU experts on packed
// 2/3-bit weights, hot experts are read from an HBM pool and the rest are
// reported as misses ("5070ti16g单卡跑qwen 3.8 flash next 新方案最高90t/s Hermes
// 调用60t/s", section "为什么从 18t/s 变成 60-90t/s"), and the always-on shared expert
// is added. With T <= 8 tokens a layer reads ~20 MB and does little
// arithmetic: it is bound by HBM and by the chain router -> top-k -> expert
// weights -> hidden -> down. Per layer:
//
//  router  every CTA bulk-copies its ~E/G router rows (and the activations)
//          into shared memory, computes those logits in the fixed fp32 order
//          and arrives at a grid barrier; meanwhile the clusters whose first
//          task is a shared-expert task start copying its weights, and every
//          CTA asks the L2 for its slice of the next layer's router rows and
//          shared expert;
//  top-k   after the barrier every CTA selects the top k of every token from
//          the logits (a CTA-wide selection, identical in all CTAs) and builds
//          the routing tables and the task list itself;
//  tasks   a task is (expert, block of HB hidden rows): HB = 128 for Q2 (one
//          block pair of the down matrix) and 256 for Q3 (one block quad).
//          The C CTAs of a cluster split a task: CTA r computes gate/up over
//          all of d for hidden rows [r HB/C, (r+1) HB/C) of the block, forms
//          h = silu(a) * u for them and pushes its h rows into every peer's
//          shared memory (st.async, completion counted in bytes on the peer's
//          mbarrier: no cluster barrier); then CTA r computes down rows
//          [r d/C, (r+1) d/C) over the block's HB columns and adds gate * y_e
//          into y with vector atomics. No task waits for another cluster. The
//          weights of a task stream into per-warp slices of a shared-memory
//          ring with bulk copies (each warp copies and waits for its own
//          bytes), the next task's copies issued as soon as a warp's slice is
//          free.
//
// Every wait on another CTA or on a copy is bounded (MOE_DEV_TIMEOUT after
// 100 ms); the last CTA to leave resets the grid counters, so the workspace
// stays zeroed between launches.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <math.h>
#include <mutex>

#include "common.cuh"
#include "layout.h"
#include "mma_q.cuh"

// Optional phase timestamps (build with -DMOE_DECODE_TRACE): thread 0 of every
// CTA records %globaltimer at each phase boundary of layer L / 2 (the only
// layer of a one-layer call) into moe_decode_trace.
#ifdef MOE_DECODE_TRACE
__device__ unsigned long long moe_decode_trace[4096 * 32];
#define TRACE(i)                                                                                      \
    do {                                                                                              \
        if (threadIdx.x == 0 && l == p.L / 2) {                                                       \
            unsigned long long t_;                                                                    \
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                                    \
            moe_decode_trace[blockIdx.x * 32 + (i)] = t_;                                             \
        }                                                                                             \
    } while (0)
// the same, recorded by lane 0 of the calling warp
#define TRACEW(i)                                                                                     \
    do {                                                                                              \
        if ((threadIdx.x & 31) == 0 && l == p.L / 2) {                                                \
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

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxTokDec = 8;
constexpr int kMaxEDec = 512;
constexpr int kMaxPairs = kMaxTokDec * kMaxK;  // 128
constexpr int kMaxDimDec = 2048;
constexpr int kMaxFDec = 4096;
constexpr unsigned long long kWaitNs = 100ull * 1000 * 1000;
constexpr unsigned long long kWaitSteps = 1ull << 27;  // polls: >= 4 s of 32 ns sleeps
constexpr int kMaxBuf = 2;                             // task buffers in the weight ring
// Copies of the logits in the workspace: every CTA reads all logits right after
// the grid barrier; CTA c reads copy c % kLogitCopies, so those reads spread
// over more L2 lines than one copy (one copy would be read by every SM at once).
constexpr int kLogitCopies = 8;

// Geometry of one launch (host-computed; see plan()).
struct Geo {
    int C;        // CTAs per cluster (hidden rows of gate/up and output rows of down split C ways)
    int HB;       // hidden rows per task (128 Q2, 256 Q3)
    int NHB;      // tasks per expert, f / HB
    int GR;       // gate/up row groups (16 rows) per CTA and task, HB / C / 16
    int RPW;      // gate/up row groups per warp (GR > 8: 2)
    int WPR;      // warps per gate/up row group (GR < 8: 8 / GR, each a share of the K quads)
    int NQ;       // 256-column quads of d
    int QPW;      // quads per warp, NQ / WPR
    int DR;       // down rows per CTA, d / C
    int NDRW;     // down row groups per warp, DR / 16 / 8
    uint32_t gu_c, gu_s;  // codes / scales bytes of one gate/up row group (one matrix, all of d)
    uint32_t dn_c, dn_s;  // codes / scales bytes of one down row group over the task's HB columns
    uint32_t gu_rg;       // one row group's gate/up bytes in a task buffer (gate codes, scales, up codes, scales)
    uint32_t gu_bytes, dn_bytes, region;  // a task buffer: GR gate/up row groups, then the down slice
    int nbuf;             // task buffers in the ring
    uint32_t red_bytes;   // per-warp gate/up results, later the down-result staging
    // dynamic shared memory offsets
    uint32_t off_bfx, off_red, off_h, off_bfh, off_ring, total;
};

struct DecodeParams {
    const uint8_t *pool;
    int64_t slot_bytes;
    int num_slots;
    int L;                       // layers in this launch
    const int32_t *slot_of;      // [L][E]
    const int32_t *shared_slot;  // [L] (device), or NULL: shared_slot0 for the one layer
    int shared_slot0;
    int layer0;                  // layer id of the first layer (miss records)
    const uint16_t *x;           // [L][T][d]
    const float *Wr;             // [L][E][d]
    const float *bias;           // [L][E] or NULL
    int T, d, f, E, k;
    float *logits;               // [2][kLogitCopies][T][E] workspace
    float *logits_out;           // [T][E] output (L == 1) or NULL
    int32_t *topk_idx;           // [L][T*k] or NULL
    float *topk_w;
    int32_t *counts, *offsets, *sorted_tok, *sorted_j, *inv, *active;  // L == 1 only (else NULL)
    int32_t *slot_of_pair;       // [L][T*k] or NULL
    moe_miss *miss;              // [L][miss_cap] or NULL
    int32_t *miss_count;         // [L] or NULL
    int miss_cap;
    int32_t *expert_counts;      // [L][E] routed pairs per expert, added to (or NULL)
    int miss_host;               // miss records / counts in mapped host memory: publish with a system fence
    float *y;                    // [L][T][d]
    int32_t *status;
    unsigned *ctr;               // [0] barrier arrivals, [1] CTAs finished
    MatGeom gate, up, down;
    Geo g;
    // the down matrix of every pool slot as [slot][row group][chunk][bytes], one
    // chunk = the codes (or scales) of one block pair (Q2) or block quad (Q3)
    CUtensorMap dn_codes, dn_scales;
};

struct Smem {
    int slot[kMaxEDec];                     // this layer's expert -> slot table
    int idx[kMaxTokDec][kMaxK];
    float w[kMaxTokDec][kMaxK];
    uint64_t wl[kWarps][kMaxK];             // per-warp top-k lists (keys)
    uint64_t sel[kMaxTokDec][kMaxK];        // merged top-k per token, best first
    float ex_r[kMaxTokDec][kMaxK];          // exp(logit - max) of the selected, by ascending id
    float inv_z[kMaxTokDec];
    float rbias[8];                         // bias of this CTA's router rows
    int pair_e[kMaxPairs];                  // expert of sorted pair s
    int s_tok[kMaxPairs], s_j[kMaxPairs];   // sorted pairs
    int inv[kMaxPairs];
    int act_e[kMaxPairs], act_beg[kMaxPairs], act_cnt[kMaxPairs], act_slot[kMaxPairs], act_mbase[kMaxPairs];
    int res[kMaxPairs];                     // active index of each resident expert
    unsigned first_mask[kMaxPairs / 32];
    float xs[kMaxDimDec / 64][kMaxTokDec];  // block sums of x over this CTA's K slice
    float hsb[4][kMaxTokDec];               // block sums of the task's h columns
    float gsel[kMaxTokDec];                 // gate of each token for the current task (0 = not routed)
    uint64_t rt_bar;                        // router rows landed
    uint64_t gu_bar[kMaxBuf][16];           // per gate/up row group of a task buffer: its bytes landed
    uint64_t dn_bar[kMaxBuf];               // the down slice of a task buffer landed
    uint64_t cand[kMaxTokDec][64];          // top-k candidates above the threshold
    int ncand[kMaxTokDec];
    uint64_t xbar[2];                       // peers' h rows landed (by task parity)
    int nact, nres, nmiss, ntask;
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

// Grid barrier arrival: this CTA's writes (ordered before it by a CTA barrier)
// are visible before the count is.
__device__ __forceinline__ void arrive_release(unsigned *ctr) {
    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(ctr) : "memory");
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

// Bulk copies global -> this CTA's shared memory that complete on an
// mbarrier (transaction bytes), and a bounded wait for an mbarrier phase.
__device__ __forceinline__ uint32_t saddr(const void *p) { return uint32_t(__cvta_generic_to_shared(p)); }
__device__ __forceinline__ void bar_init(uint64_t *bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(saddr(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void bar_expect(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(saddr(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bulk_copy(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     saddr(dst)),
                 "l"(src), "r"(bytes), "r"(saddr(bar))
                 : "memory");
}
__device__ __forceinline__ bool bar_test(uint64_t *bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n.reg .pred q;\nmbarrier.try_wait.parity.shared::cta.b64 q, [%1], %2;\nselp.u32 %0, 1, 0, q;\n}"
        : "=r"(done)
        : "r"(saddr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}
// false after kWaitNs, or kWaitSteps polls (the caller flags MOE_DEV_TIMEOUT)
__device__ bool bar_wait(uint64_t *bar, uint32_t parity) {
    if (bar_test(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    for (unsigned long long it = 0; !bar_test(bar, parity); ++it) {
        if (globaltimer() - t0 > kWaitNs || it > kWaitSteps) return false;
        if (it > 1024) __nanosleep(32);
    }
    return true;
}

// Cluster helpers: this CTA's rank, and every thread's arrival + wait at the
// cluster barrier (hardware; each CTA of a cluster runs the same sequence of
// cluster barriers on every path, so each one completes).
__device__ __forceinline__ unsigned cluster_rank() {
    unsigned r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ unsigned cluster_id() {
    unsigned r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}
__device__ __forceinline__ unsigned cluster_count() {
    unsigned r;
    asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address of the same shared-memory object in cluster CTA `rank`.
__device__ __forceinline__ uint32_t peer_addr(const void *p, unsigned rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr(p)), "r"(rank));
    return r;
}
// 16 bytes into a peer CTA's shared memory, counted on the peer's mbarrier.
__device__ __forceinline__ void st_async4(uint32_t raddr, float4 v, uint32_t rbar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1,%2,%3,%4}, [%5];" ::"r"(raddr),
                 "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w), "r"(rbar)
                 : "memory");
}
__device__ __forceinline__ void red_add4(float *p, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1,%2,%3,%4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
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
    bar_init(&bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    if (!bar_wait(&bar, 0u)) flag(status, MOE_DEV_TIMEOUT);
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
__device__ __forceinline__ float key_value(uint32_t key) {
    return __uint_as_float((key & 0x80000000u) ? (key ^ 0x80000000u) : ~key);
}

// One router row (fixed fp32 order, see moe.h) for NT tokens from shared memory.
template <int NT>
__device__ void router_row(const float *wrow, const uint16_t *sx, int T, int d, int lane, bool has_bias, float b,
                           int e, float *logits, float *logits_out, int E, int32_t *status) {
    float acc[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[t] = 0.f;
    for (int u = 0; u < d / 128; ++u) {
        const float4 wv = *reinterpret_cast<const float4 *>(wrow + 128 * u + 4 * lane);
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            if (t < T) {
                const uint2 xv = *reinterpret_cast<const uint2 *>(sx + size_t(t) * d + 128 * u + 4 * lane);
                float a = acc[t];
                a = __fmaf_rn(bf16_lo(xv.x), wv.x, a);
                a = __fmaf_rn(bf16_hi(xv.x), wv.y, a);
                a = __fmaf_rn(bf16_lo(xv.y), wv.z, a);
                a = __fmaf_rn(bf16_hi(xv.y), wv.w, a);
                acc[t] = a;
            }
        }
    }
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) acc[t] = __fadd_rn(acc[t], __shfl_xor_sync(0xffffffffu, acc[t], o));
    if (lane < kLogitCopies) {  // lane c writes copy c
        for (int t = 0; t < T; ++t) {
            const float v = has_bias ? __fadd_rn(acc[t], b) : acc[t];
            if (lane == 0 && !isfinite(v)) flag(status, MOE_DEV_NONFINITE);
            __stcg(logits + (size_t(lane) * T + t) * E + e, v);
            if (lane == 0 && logits_out) logits_out[size_t(t) * E + e] = v;
        }
    }
}

// One 64-weight block of a 16-row tile against B (4 MMAs over k 0..63) as two
// independent chains of two MMAs (k 0..31 and 32..63) summed at the end.
template <int FMT>
__device__ __forceinline__ void block_mma(const QuadRegs<FMT> &q, int bq, const uint32_t (&Bb)[8], float (&c)[4]) {
    float p[2][4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t a0, a1, a2, a3;
        if constexpr (FMT == 2) {
            const uint32_t wg = bq == 0 ? q.c0.x : bq == 1 ? q.c0.z : bq == 2 ? q.c1.x : q.c1.z;
            const uint32_t wg8 = bq == 0 ? q.c0.y : bq == 1 ? q.c0.w : bq == 2 ? q.c1.y : q.c1.w;
            a0 = q2_reg(wg, 2 * i);
            a1 = q2_reg(wg8, 2 * i);
            a2 = q2_reg(wg, 2 * i + 1);
            a3 = q2_reg(wg8, 2 * i + 1);
        } else {
            const int u0 = 8 * bq + 2 * i, u1 = u0 + 1;
            a0 = q3_reg(q.W, u0, 0);
            a1 = q3_reg(q.W, u0, 1);
            a2 = q3_reg(q.W, u1, 0);
            a3 = q3_reg(q.W, u1, 1);
        }
        if (i < 2)
            mma16816_zc(p[i], a0, a1, a2, a3, Bb[2 * i], Bb[2 * i + 1]);
        else
            mma16816(p[i - 2], a0, a1, a2, a3, Bb[2 * i], Bb[2 * i + 1]);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) c[j] = p[0][j] + p[1][j];
}

template <int FMT>
__device__ __forceinline__ uint32_t block_scale(const QuadRegs<FMT> &q, int bq) {
    if constexpr (FMT == 2) return bq == 0 ? q.s0.x : bq == 1 ? q.s0.z : bq == 2 ? q.s1.x : q.s1.z;
    else return bq == 0 ? q.s0.x : bq == 1 ? q.s0.y : bq == 2 ? q.s1.x : q.s1.y;
}
template <int FMT>
__device__ __forceinline__ uint32_t block_min(const QuadRegs<FMT> &q, int bq) {
    if constexpr (FMT == 2) return bq == 0 ? q.s0.y : bq == 1 ? q.s0.w : bq == 2 ? q.s1.y : q.s1.w;
    else return 0u;
}

// Gate and up tiles of one 16-row x 256-column quad against the same B,
// block by block with the two matrices interleaved (8 independent MMAs per block).
template <int FMT>
__device__ __forceinline__ void quad_pair_compute(const QuadRegs<FMT> &qg, const QuadRegs<FMT> &qu,
                                                  const uint32_t (&B)[4][8], const float (&xs)[4][2],
                                                  float (&ag)[4], float (&au)[4]) {
#pragma unroll
    for (int bq = 0; bq < 4; ++bq) {
        float cg[4], cu[4];
        block_mma<FMT>(qg, bq, B[bq], cg);
        block_mma<FMT>(qu, bq, B[bq], cu);
        block_epilogue<FMT>(cg, block_scale<FMT>(qg, bq), block_min<FMT>(qg, bq), xs[bq][0], xs[bq][1], ag);
        block_epilogue<FMT>(cu, block_scale<FMT>(qu, bq), block_min<FMT>(qu, bq), xs[bq][0], xs[bq][1], au);
    }
}

// One quad (4 blocks) of one matrix.
template <int FMT>
__device__ __forceinline__ void quad_compute_ilp(const QuadRegs<FMT> &q, const uint32_t (&B)[4][8],
                                                 const float (&xs)[4][2], float (&acc)[4]) {
    float c[4][4];
#pragma unroll
    for (int bq = 0; bq < 4; ++bq) block_mma<FMT>(q, bq, B[bq], c[bq]);
#pragma unroll
    for (int bq = 0; bq < 4; ++bq)
        block_epilogue<FMT>(c[bq], block_scale<FMT>(q, bq), block_min<FMT>(q, bq), xs[bq][0], xs[bq][1], acc);
}

// Q2 down tiles of one block pair (16 rows x 128 columns) for two row groups:
// c = a lane's 16 code bytes, s = its 16 scale bytes (see layout.h), B / xs of
// the pair's two blocks; 16 independent MMAs.
__device__ __forceinline__ void pair2_compute_q2(uint4 c0, uint4 s0, uint4 c1, uint4 s1, const uint32_t (&B)[2][8],
                                                 const float (&xs)[2][2], float (&acc0)[4], float (&acc1)[4]) {
    QuadRegs<2> q0, q1;  // blocks 0, 1 of each pair in the first half of a quad's registers
    q0.c0 = c0;
    q0.s0 = s0;
    q1.c0 = c1;
    q1.s0 = s1;
    q0.c1 = q1.c1 = make_uint4(0u, 0u, 0u, 0u);
    q0.s1 = q1.s1 = make_uint4(0u, 0u, 0u, 0u);
    float r[4][4];
    block_mma<2>(q0, 0, B[0], r[0]);
    block_mma<2>(q0, 1, B[1], r[1]);
    block_mma<2>(q1, 0, B[0], r[2]);
    block_mma<2>(q1, 1, B[1], r[3]);
    block_epilogue<2>(r[0], s0.x, s0.y, xs[0][0], xs[0][1], acc0);
    block_epilogue<2>(r[1], s0.z, s0.w, xs[1][0], xs[1][1], acc0);
    block_epilogue<2>(r[2], s1.x, s1.y, xs[0][0], xs[0][1], acc1);
    block_epilogue<2>(r[3], s1.z, s1.w, xs[1][0], xs[1][1], acc1);
}

// Packed codes and scales of one 16-row x 256-column tile from shared memory:
// cb / sb point at the first quad of a row group's slice as copied from the
// record (codes contiguous per quad, scales per block pair).
template <int FMT>
__device__ __forceinline__ void quad_smem(const uint8_t *cb, const uint8_t *sb, int qi, int lane, QuadRegs<FMT> &q) {
    const int g = lane >> 2;
    if constexpr (FMT == 2) {
        q.c0 = *reinterpret_cast<const uint4 *>(cb + ((2 * qi) * 32 + lane) * 16);
        q.c1 = *reinterpret_cast<const uint4 *>(cb + ((2 * qi + 1) * 32 + lane) * 16);
        q.s0 = *reinterpret_cast<const uint4 *>(sb + ((2 * qi) * 8 + g) * 16);
        q.s1 = *reinterpret_cast<const uint4 *>(sb + ((2 * qi + 1) * 8 + g) * 16);
    } else {
#pragma unroll
        for (int w = 0; w < 3; ++w) {
            const uint4 v = *reinterpret_cast<const uint4 *>(cb + qi * 1536 + w * 512 + lane * 16);
            q.W[4 * w + 0] = v.x;
            q.W[4 * w + 1] = v.y;
            q.W[4 * w + 2] = v.z;
            q.W[4 * w + 3] = v.w;
        }
        q.s0 = *reinterpret_cast<const uint2 *>(sb + ((2 * qi) * 8 + g) * 8);
        q.s1 = *reinterpret_cast<const uint2 *>(sb + ((2 * qi + 1) * 8 + g) * 8);
    }
}

// Per-layer pointers.
struct LayerPtrs {
    const int32_t *slot_of;
    const uint16_t *x;
    const float *Wr, *bias;
    float *y, *logits;  // logits: this layer's copies in the workspace
    int shared_slot;
};
__device__ __forceinline__ LayerPtrs layer_ptrs(const DecodeParams &p, int l) {
    LayerPtrs q;
    q.slot_of = p.slot_of + size_t(l) * p.E;
    q.x = p.x + size_t(l) * p.T * p.d;
    q.Wr = p.Wr + size_t(l) * p.E * p.d;
    q.bias = p.bias ? p.bias + size_t(l) * p.E : nullptr;
    q.y = p.y + size_t(l) * p.T * p.d;
    q.logits = p.logits + size_t(l & 1) * kLogitCopies * p.T * p.E;
    q.shared_slot = p.shared_slot ? __ldg(p.shared_slot + l) : p.shared_slot0;
    return q;
}

// Task tau of the layer: the shared expert's blocks first, then the resident
// routed experts' blocks. Returns the pool slot, sets hb and the active index
// (-1 for the shared expert).
__device__ __forceinline__ int task_slot(const DecodeParams &p, const Smem &s, const LayerPtrs &lp, int tau, int &hb,
                                         int &a) {
    const int NHB = p.g.NHB;
    if (tau < NHB) {
        hb = tau;
        a = -1;
        return lp.shared_slot;
    }
    const int r = (tau - NHB) / NHB;
    hb = (tau - NHB) % NHB;
    a = s.res[r];
    return s.act_slot[a];
}

// Gate/up row group (task-local, 0 .. GR-1) and first quad of warp `warp`'s
// ri-th share of the task.
__device__ __forceinline__ int gu_rgl(const Geo &g, int warp, int ri) { return g.WPR > 1 ? warp / g.WPR : warp + 8 * ri; }
__device__ __forceinline__ int gu_q0(const Geo &g, int warp) { return g.QPW * (warp % g.WPR); }

__device__ __forceinline__ void tma_load_4d(void *dst, const CUtensorMap *map, int c0, int c1, int c2, int c3,
                                            uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, "
        "%5}], [%6];" ::"r"(saddr(dst)),
        "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(saddr(bar))
        : "memory");
}

// Copies of task (slot, hb) into buffer b: for each of its GR gate/up row
// groups, the gate and up codes and scales over all of d (4 bulk copies,
// completing on that row group's barrier). Copy c is issued by lane c / 8 of
// warp c % 8, so the copies of a task leave from all warps at once.
template <int FMT>
__device__ __noinline__ void issue_gu(const DecodeParams &p, Smem &s, uint8_t *ring, int b, int tid, unsigned rank,
                                      int slot, int hb) {
    const Geo &g = p.g;
    const int c = (tid & 31) * kWarps + (tid >> 5);
    if (c >= 4 * g.GR) return;
    const int rgl = c >> 2, mi = (c >> 1) & 1, sc = c & 1;
    const uint8_t *rec = p.pool + int64_t(slot) * p.slot_bytes;
    const MatGeom &m = mi ? p.up : p.gate;
    const int rg = hb * (g.HB / 16) + int(rank) * g.GR + rgl;
    uint8_t *dst = ring + size_t(b) * g.region + size_t(rgl) * g.gu_rg + size_t(mi) * (g.gu_c + g.gu_s) +
                   (sc ? g.gu_c : 0);
    if ((c & 3) == 0) bar_expect(&s.gu_bar[b][rgl], g.gu_rg);
    const uint64_t off = sc ? scale_off(m, FMT, rg, 0, 0) : (FMT == 2 ? q2_chunk_off(m, rg, 0, 0) : q3_word_off(m, rg, 0, 0, 0));
    bulk_copy(dst, rec + off, sc ? g.gu_s : g.gu_c, &s.gu_bar[b][rgl]);
}

// The down slice of task (slot, hb) into buffer b, by thread 0: this CTA's DR
// rows over the task's HB columns (block pair hb for Q2, block quad hb for
// Q3), codes then scales, as two tensor copies.
__device__ __noinline__ void issue_dn(const DecodeParams &p, Smem &s, uint8_t *ring, int b, int tid, unsigned rank,
                                      int slot, int hb) {
    const Geo &g = p.g;
    if (tid != 0) return;
    uint8_t *dst = ring + size_t(b) * g.region + g.gu_bytes;
    const int ndr = g.DR / 16;
    bar_expect(&s.dn_bar[b], g.dn_bytes);
    tma_load_4d(dst, &p.dn_codes, 0, hb, int(rank) * ndr, slot, &s.dn_bar[b]);
    tma_load_4d(dst + size_t(ndr) * g.dn_c, &p.dn_scales, 0, hb, int(rank) * ndr, slot, &s.dn_bar[b]);
}

// k largest of a warp's M keys per lane (64-bit: logit key << 32 | ~id),
// descending, by k rounds of a warp-wide maximum; lane r < k receives the r-th.
template <int M>
__device__ __forceinline__ uint64_t warp_topk(uint64_t (&c)[M], int k, int lane) {
    uint64_t mine = 0ull;
    for (int r = 0; r < k; ++r) {
        uint64_t mx = 0ull;
#pragma unroll
        for (int m = 0; m < M; ++m) mx = c[m] > mx ? c[m] : mx;
        const uint32_t hk = __reduce_max_sync(0xffffffffu, uint32_t(mx >> 32));
        const uint32_t lk = __reduce_max_sync(0xffffffffu, uint32_t(mx >> 32) == hk ? uint32_t(mx) : 0u);
        const uint64_t win = (uint64_t(hk) << 32) | lk;
        if (lane == r) mine = win;
        if (mx == win && win != 0ull) {
#pragma unroll
            for (int m = 0; m < M; ++m)
                if (c[m] == win) c[m] = 0ull;
        }
    }
    return mine;
}

// Near-equal logits (more than 64 keys reach the threshold): every warp finds
// its exact top k by rounds and each token's lists are merged by counting.
template <int NT, int M>
__device__ __noinline__ void topk_exact(Smem &s, const uint64_t (&orig)[M], bool many, int k) {
    constexpr int WPT = kWarps / NT;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int tt = warp / WPT;
    if (many) {
        uint64_t c[M];
#pragma unroll
        for (int m = 0; m < M; ++m) c[m] = orig[m];
        const uint64_t mine = warp_topk<M>(c, k, lane);
        if (lane < k) s.wl[warp][lane] = mine;
    }
    __syncthreads();
    if (many && lane < k) {
        const uint64_t me = s.wl[warp][lane];
        int rank = 0;
        for (int o = 0; o < WPT; ++o)
            for (int q = 0; q < k; ++q) rank += s.wl[tt * WPT + o][q] > me;
        if (rank < k) s.sel[tt][rank] = me;
    }
}

// Top-k of every token from the logits in global memory (written by all CTAs
// of this launch). A candidate is the 64-bit key (logit key << 32 | ~id), so
// the top k are the k largest keys (larger logit first, then lower id).
// WPT = 8 / NT warps share a token's experts. With WPT > 1 each warp finds the
// R-th largest of its keys (R = ceil(k / WPT) rounds of a warp-wide maximum);
// the smallest of those, L, has at least R * WPT >= k keys at or above it, so
// the top k are the k largest of the keys >= L (usually a few dozen), ranked
// by counting. If more than 64 keys reach L (near-equal logits) every warp
// finds its exact top k by rounds and the lists are merged by counting. With
// WPT = 1 the warp's k rounds give the answer. Then softmax over the selected
// logits in ascending-id order (the arithmetic of moe_route).
template <int NT>
__device__ __noinline__ void topk_cta(const DecodeParams &p, Smem &s, const float *logits, int T, int E, int k) {
    constexpr int WPT = kWarps / NT;       // warps per token
    constexpr int M = kMaxEDec / 32 / WPT;  // keys per lane
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int tt = warp / WPT, sub = warp % WPT;
    uint64_t c[M], orig[WPT > 1 ? M : 1];
    if (tid < kMaxTokDec) s.ncand[tid] = 0;
    const int l = p.L / 2;  // (trace points of the traced layer only; the caller passes that layer's logits)
    (void)l;
    if (tt < T) {
        const float *row = logits + size_t(tt) * E;
        bool nan = false;
#pragma unroll
        for (int m = 0; m < M; ++m) {
            const int e = sub * 32 + lane + 32 * WPT * m;
            if (e < E) {
                const float v = __ldcg(row + e);
                nan |= v != v;
                c[m] = (uint64_t(logit_key(v)) << 32) | uint64_t(~uint32_t(e));
            } else {
                c[m] = 0ull;
            }
            if constexpr (WPT > 1) orig[m] = c[m];
        }
        if (__any_sync(0xffffffffu, nan) && lane == 0 && blockIdx.x == 0) flag(p.status, MOE_DEV_NONFINITE);
        TRACE(14);
        if constexpr (WPT == 1) {
            const uint64_t mine = warp_topk<M>(c, k, lane);
            if (lane < k) s.sel[tt][lane] = mine;
        } else {
            const int R = (k + WPT - 1) / WPT;
            const uint64_t mine = warp_topk<M>(c, R, lane);
            if (lane == R - 1) s.wl[warp][0] = mine;  // this warp's R-th largest
        }
    }
    if constexpr (WPT > 1) {
        __syncthreads();
        TRACE(15);
        if (tt < T) {  // gather the keys >= L
            uint64_t L = ~0ull;
#pragma unroll
            for (int o = 0; o < WPT; ++o) {
                const uint64_t v = s.wl[tt * WPT + o][0];
                L = v < L ? v : L;
            }
#pragma unroll
            for (int m = 0; m < M; ++m) {
                const bool in = orig[m] != 0ull && orig[m] >= L;
                const unsigned bal = __ballot_sync(0xffffffffu, in);
                int base = 0;
                if (lane == 0 && bal) base = atomicAdd(&s.ncand[tt], __popc(bal));
                base = __shfl_sync(0xffffffffu, base, 0);
                const int pos = base + __popc(bal & ((1u << lane) - 1u));
                if (in && pos < 64) s.cand[tt][pos] = orig[m];
            }
        }
        __syncthreads();
        TRACE(16);
        const bool many = tt < T && s.ncand[tt] > 64;
        if (tt < T && !many) {  // rank the candidates: keys above mine
            const int n = s.ncand[tt];
            for (int i = sub * 32 + lane; i < n; i += WPT * 32) {
                const uint64_t me = s.cand[tt][i];
                int rank = 0;
#pragma unroll 4
                for (int q = 0; q < n; ++q) rank += s.cand[tt][q] > me;
                if (rank < k) s.sel[tt][rank] = me;
            }
        }
        if (__syncthreads_or(many)) topk_exact<NT, M>(s, orig, many, k);
    }
    __syncthreads();
    TRACE(17);
    // softmax over the selected logits in ascending-id order (the arithmetic of
    // moe_route: z summed from 0 in that order, gate = ex * (1 / z))
    const bool selt = warp < T && lane < k;
    int my_id = 0, rank = 0;
    float ex = 0.f;
    if (selt) {
        const uint64_t mine = s.sel[warp][lane];
        const uint32_t key = uint32_t(mine >> 32);
        // a round that found only NaN left takes expert 0 with logit -inf, as moe_route does
        my_id = key ? int(~uint32_t(mine)) : 0;
        const float my_v = key ? key_value(key) : -INFINITY;
        const uint64_t top = s.sel[warp][0];
        const float mx = uint32_t(top >> 32) ? key_value(uint32_t(top >> 32)) : -INFINITY;
#pragma unroll 4
        for (int q = 0; q < kMaxK; ++q) {
            if (q < k) {
                const uint64_t o = s.sel[warp][q];
                const int oid = uint32_t(o >> 32) ? int(~uint32_t(o)) : 0;
                rank += oid < my_id;
            }
        }
        ex = expf(my_v - mx);
        s.ex_r[warp][rank] = ex;
    }
    __syncthreads();
    if (warp < T && lane == 0) {
        float z = 0.0f;
        for (int a = 0; a < k; ++a) z += s.ex_r[warp][a];
        s.inv_z[warp] = 1.0f / z;
    }
    __syncthreads();
    if (selt) {
        s.idx[warp][rank] = my_id;
        s.w[warp][rank] = ex * s.inv_z[warp];
    }
    __syncthreads();
}

// Routing tables from s.idx: sorted pairs, active experts with their slots,
// resident list, miss bases, and the task count. Whole CTA.
__device__ __noinline__ void routing_tables(const DecodeParams &p, Smem &s, int T, int k) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int npairs = T * k;
    if (T == 1) {  // one token: its k experts (ascending id) are the active experts, one pair each
        if (warp == 0) {
            const bool in = lane < k;
            int sl = -1;
            if (in) {
                const int e = s.idx[0][lane];
                s.pair_e[lane] = e;
                s.s_tok[lane] = 0;
                s.s_j[lane] = lane;
                s.inv[lane] = lane;
                sl = (e >= 0 && e < p.E) ? s.slot[e] : -1;
                const bool bad = sl < -1 || sl >= p.num_slots;
                if (bad && blockIdx.x == 0) flag(p.status, MOE_DEV_BAD_SLOT);
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
                s.ntask = (__popc(rm) + 1) * p.g.NHB;
            }
        }
        __syncthreads();
        return;
    }
    if (tid < npairs) s.pair_e[tid] = s.idx[tid / k][tid % k];  // flat ids (pair p = t*k + j)
    __syncthreads();
    int my_e = 0, my_rank = 0;
    if (tid < npairs) {  // stable sort of the pairs by (expert, pair index)
        my_e = s.pair_e[tid];
#pragma unroll 4
        for (int q = 0; q < npairs; ++q) {
            const int eq = s.pair_e[q];
            my_rank += (eq < my_e) || (eq == my_e && q < tid);
        }
    }
    __syncthreads();
    if (tid < npairs) {
        const int t = tid / k;
        s.pair_e[my_rank] = my_e;
        s.s_tok[my_rank] = t;
        s.s_j[my_rank] = tid - t * k;
        s.inv[tid] = my_rank;
    }
    __syncthreads();
    const bool in = tid < npairs;
    const bool first = in && (tid == 0 || s.pair_e[tid] != s.pair_e[tid - 1]);
    const unsigned fm = __ballot_sync(0xffffffffu, first);
    if (lane == 0 && warp < kMaxPairs / 32) s.first_mask[warp] = fm;
    __syncthreads();
    if (first) {
        int a = __popc(fm & ((1u << lane) - 1));
        for (int w = 0; w < warp; ++w) a += __popc(s.first_mask[w]);
        const int e = s.pair_e[tid];
        const int sl = (e >= 0 && e < p.E) ? s.slot[e] : -1;
        const bool bad = sl < -1 || sl >= p.num_slots;
        if (bad && blockIdx.x == 0) flag(p.status, MOE_DEV_BAD_SLOT);
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
            s.ntask = (nr + 1) * p.g.NHB;
        }
    }
    __syncthreads();
}

// Routing, permutation, slots and misses of layer l to global memory (one CTA).
__device__ __noinline__ void publish(const DecodeParams &p, Smem &s, int l, int T, int k, int E) {
    const int tid = threadIdx.x;
    const int npairs = T * k;
    const size_t po = size_t(l) * npairs;
    for (int i = tid; i < npairs; i += kThreads) {
        const int t = i / k, j = i % k;
        if (p.topk_idx) p.topk_idx[po + i] = s.idx[t][j];
        if (p.topk_w) p.topk_w[po + i] = s.w[t][j];
        if (p.sorted_tok) p.sorted_tok[i] = s.s_tok[i];
        if (p.sorted_j) p.sorted_j[i] = s.s_j[i];
        if (p.inv) p.inv[i] = s.inv[i];
    }
    if (p.offsets || p.counts) {
        for (int e = tid; e <= E; e += kThreads) {
            int lo = 0, hi = s.nact;  // first active expert >= e
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if (s.act_e[mid] < e) lo = mid + 1; else hi = mid;
            }
            if (p.offsets) p.offsets[e] = lo < s.nact ? s.act_beg[lo] : npairs;
            if (p.counts && e < E) p.counts[e] = (lo < s.nact && s.act_e[lo] == e) ? s.act_cnt[lo] : 0;
        }
    }
    if (p.active) {
        for (int a = tid; a < s.nact; a += kThreads) p.active[1 + a] = s.act_e[a];
        if (tid == 0) p.active[0] = s.nact;
    }
    if (p.expert_counts)
        for (int i = tid; i < npairs; i += kThreads) atomicAdd(p.expert_counts + size_t(l) * E + s.idx[i / k][i % k], 1);
    moe_miss *miss = p.miss ? p.miss + size_t(l) * p.miss_cap : nullptr;
    for (int sp = tid; sp < npairs; sp += kThreads) {
        int a = 0;
        while (a + 1 < s.nact && s.act_beg[a + 1] <= sp) ++a;
        const bool res = s.act_slot[a] >= 0;
        const int pp = s.s_tok[sp] * k + s.s_j[sp];
        if (p.slot_of_pair) p.slot_of_pair[po + pp] = res ? s.act_slot[a] : -1;
        if (!res && miss) {
            const int mi = s.act_mbase[a] + (sp - s.act_beg[a]);
            if (mi < p.miss_cap) {
                moe_miss m;
                m.layer = p.layer0 + l;
                m.expert = s.act_e[a];
                m.token = s.s_tok[sp];
                m.j = s.s_j[sp];
                m.gate = s.w[m.token][m.j];
                miss[mi] = m;
            }
        }
    }
    // the count last, after every record is visible system-wide: a host reader of
    // mapped memory that sees the count sees the records (device readers run
    // after the kernel and need no fence)
    __syncthreads();
    if (tid == 0) {
        if (p.miss_host) __threadfence_system();
        if (p.miss_count) *reinterpret_cast<volatile int32_t *>(p.miss_count + l) = s.nmiss;
        if (s.nmiss > p.miss_cap && p.miss) flag(p.status, MOE_DEV_MISS_OVERFLOW);
    }
}

template <int FMT, int NT>
__global__ void __launch_bounds__(kThreads, 1) decode_layer_kernel(const __grid_constant__ DecodeParams p) {
    extern __shared__ __align__(128) unsigned char dyn[];
    __shared__ Smem s;
    const Geo &g = p.g;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = gridDim.x, cta = blockIdx.x;
    const unsigned rank = cluster_rank(), cid = cluster_id(), ncl = cluster_count();
    const int T = p.T, k = p.k, E = p.E, d = p.d;
    const int gl = lane >> 2, tl = lane & 3;  // MMA fragment coordinates of this lane
    uint4 *bfx = reinterpret_cast<uint4 *>(dyn + g.off_bfx);  // x B fragments [NQ][8][NT*4] (lanes g < NT)
    float *red = reinterpret_cast<float *>(dyn + g.off_red);  // [8 warps][RPW][32][8] gate/up results; down staging
    float *hs_all = reinterpret_cast<float *>(dyn + g.off_h);  // [2][HB][NT] h of the task (by task parity)
    uint32_t *bfh = reinterpret_cast<uint32_t *>(dyn + g.off_bfh);  // [HB/64][8][32] h B fragments
    uint8_t *ring = dyn + g.off_ring;
    bool too_big = false, ok = true;
    unsigned bar_target = 0;  // grid barrier arrivals this CTA has waited for
    int seq = 0;  // tasks of this CTA started so far, over all layers (buffer = seq % nbuf, h parity = seq % 2)

    if (tid == 0) {
        bar_init(&s.rt_bar, 1);
        for (int b = 0; b < kMaxBuf; ++b) {
            for (int r = 0; r < 16; ++r) bar_init(&s.gu_bar[b][r], 1);
            bar_init(&s.dn_bar[b], 1);
        }
        bar_init(&s.xbar[0], 1);
        bar_init(&s.xbar[1], 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // every CTA of the cluster has initialised its barriers before a peer sends to them
    cluster_sync();

    // rows of the router this CTA computes (contiguous, about E/G)
    const int rb = int(int64_t(E) * cta / G), re = int(int64_t(E) * (cta + 1) / G);
    const int nrows = re - rb;

#ifdef MOE_DECODE_TRACE
    if (tid == 0) {  // points this launch does not reach stay empty; 30/31: SM cycles at start / end
        for (int i = 1; i < 32; ++i) moe_decode_trace[blockIdx.x * 32 + i] = 0ull;
        moe_decode_trace[blockIdx.x * 32 + 30] = clock64();
    }
#endif
    for (int l = 0; l < p.L; ++l) {
        const LayerPtrs lp = layer_ptrs(p, l);
        TRACE(0);
        // ------------------------------------------------ router rows + activations
        float *rrows = reinterpret_cast<float *>(ring);  // router rows, then x, in the ring
        uint16_t *sx = reinterpret_cast<uint16_t *>(ring + size_t(nrows) * d * 4);
        // layers after the first had their router rows and x staged at the end of
        // the previous layer (while its grid barrier was pending)
        if (l == 0 && tid == 0 && nrows > 0) {
            bar_expect(&s.rt_bar, uint32_t(nrows) * uint32_t(d) * 4u);
            bulk_copy(rrows, lp.Wr + size_t(rb) * d, uint32_t(nrows) * uint32_t(d) * 4u, &s.rt_bar);
        }
        {
            if (tid < nrows && tid < 8) s.rbias[tid] = lp.bias ? __ldg(lp.bias + rb + tid) : 0.f;
            const uint4 *src = reinterpret_cast<const uint4 *>(lp.x);
            uint4 *dst = reinterpret_cast<uint4 *>(sx);
            for (int i = tid; l == 0 && i < T * d / 8; i += kThreads) dst[i] = __ldg(src + i);
            for (int e = tid; e < E; e += kThreads) s.slot[e] = __ldg(lp.slot_of + e);
            // this CTA's slice of y starts at zero (before the grid barrier, so before any atomic)
            for (int i = cta * kThreads + tid; i < T * d; i += G * kThreads) lp.y[i] = 0.f;
        }
        __syncthreads();
        TRACE(12);
        // block sums of x and its B fragments (token columns < NT; the rest are zero)
        for (int job = warp; job < (d / 64) * T; job += kWarps) {
            const int bb = job / T, n = job % T;
            const uint32_t u = *reinterpret_cast<const uint32_t *>(sx + size_t(n) * d + 64 * bb + 2 * lane);
            float v = bf16_lo(u) + bf16_hi(u);
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == 0) s.xs[bb][n] = v;
        }
        for (int e = tid; e < g.NQ * 8 * NT * 4; e += kThreads) {
            const int qi = e / (8 * NT * 4), r4 = (e / (NT * 4)) % 8, ln = e % (NT * 4);
            const int gg = ln >> 2, tt = ln & 3, bq = r4 >> 1;
            const uint16_t *src = sx + size_t(gg) * d + 256 * qi + 64 * bq;
            uint32_t v[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int rho = (r4 & 1) * 4 + j;
                float lo = 0.f, hi = 0.f;
                if (gg < T) {
                    const uint32_t u = *reinterpret_cast<const uint32_t *>(src + slot_k(rho, tt, 0));
                    lo = bf16_lo(u);
                    hi = bf16_hi(u);
                }
                const float sc = __int_as_float((127 - slot_exp<FMT>(bq, rho)) << 23);  // 2^-exp
                v[j] = pack_half2(lo * sc, hi * sc);
            }
            bfx[e] = make_uint4(v[0], v[1], v[2], v[3]);
        }
        if (nrows > 0) {
            const bool got = bar_wait(&s.rt_bar, uint32_t(l & 1));
            if (!got && tid == 0) flag(p.status, MOE_DEV_TIMEOUT);
            ok = ok && got;
            TRACE(13);
            for (int r = warp; got && r < nrows; r += kWarps)
                router_row<NT>(rrows + size_t(r) * d, sx, T, d, lane, lp.bias != nullptr,
                               r < 8 ? s.rbias[r] : (lp.bias ? __ldg(lp.bias + rb + r) : 0.f), rb + r, lp.logits,
                               p.logits_out, E, p.status);
        }
        ok = __syncthreads_and(ok) != 0;  // logits written; router rows and x consumed (the ring is free)
        if (tid == 0) arrive_release(p.ctr);
        bar_target += unsigned(G);
        TRACE(1);
        // this cluster's tasks known before routing: the shared expert's blocks
        const int nsh = g.NHB;
        int known = 0;  // tasks of this cluster whose index is known (its list: cid, cid + ncl, ...)
        while (int(cid) + known * int(ncl) < nsh) ++known;
        const int seq0 = seq;  // this layer's first task of this CTA
        int gu_next = 0, dn_next = 0;  // next task (layer-local) whose copies are issued (CTA-uniform)
        // called by every thread at the same points, after a CTA barrier that
        // frees the buffers being refilled
        auto issue_upto = [&](int n_known, int gu_done, int dn_done) {
            while (gu_next < n_known && gu_next < gu_done + g.nbuf) {
                int hb, a;
                const int slot = task_slot(p, s, lp, int(cid) + gu_next * int(ncl), hb, a);
                issue_gu<FMT>(p, s, ring, (seq0 + gu_next) % g.nbuf, tid, rank, slot, hb);
                ++gu_next;
            }
            while (dn_next < n_known && dn_next < dn_done + g.nbuf) {
                int hb, a;
                const int slot = task_slot(p, s, lp, int(cid) + dn_next * int(ncl), hb, a);
                issue_dn(p, s, ring, (seq0 + dn_next) % g.nbuf, tid, rank, slot, hb);
                ++dn_next;
            }
        };
        if (ok) issue_upto(known, 0, 0);
        // the next layer's router rows and a slice of its shared expert into the L2
        if (tid == 0 && l + 1 < p.L) {
            const LayerPtrs np = layer_ptrs(p, l + 1);
            if (nrows > 0) prefetch_l2(np.Wr + size_t(rb) * d, uint32_t(nrows) * uint32_t(d) * 4u);
            const uint64_t eb = uint64_t(p.down.codes_off) + p.down.bytes;  // record bytes
            const uint64_t c0 = (eb * uint64_t(cta) / uint64_t(G)) & ~uint64_t(15);
            const uint64_t c1 = (eb * uint64_t(cta + 1) / uint64_t(G)) & ~uint64_t(15);
            if (c1 > c0) prefetch_l2(p.pool + int64_t(np.shared_slot) * p.slot_bytes + c0, uint32_t(c1 - c0));
            if (cta == 0) prefetch_l2(np.slot_of, uint32_t(E) * 4u);
            if (cta == 1) prefetch_l2(np.x, uint32_t(T) * uint32_t(d) * 2u);
        }
        // ------------------------------------------------ grid barrier: all logits written
        if (tid == 0) s.ok = wait_geq(p.ctr, bar_target, p.status);
        __syncthreads();
        ok = ok && s.ok;
        TRACE(2);
        if (ok) {
            topk_cta<NT>(p, s, lp.logits + size_t(cta % kLogitCopies) * T * E, T, E, k);
            TRACE(3);
            routing_tables(p, s, T, k);
        }
        TRACE(4);
        // every CTA of a cluster derives the same task list from the same routing;
        // a CTA that could not route runs none (its peers' waits for it give up)
        const int ntask = ok ? s.ntask : 0;
        const int nmine = ntask > int(cid) ? (ntask - int(cid) + int(ncl) - 1) / int(ncl) : 0;
        if (ok) issue_upto(nmine, 0, 0);
        TRACE(11);
        // ------------------------------------------------ tasks
        const int hrows = g.GR * 16;  // hidden rows this CTA computes per task
        for (int i = 0; i < nmine; ++i) {
            const int b = (seq0 + i) % g.nbuf;
            const uint32_t ph = uint32_t((seq0 + i) / g.nbuf) & 1u;
            const int xb = (seq0 + i) & 1;
            const uint32_t xph = uint32_t((seq0 + i) >> 1) & 1u;
            float *hs = hs_all + size_t(xb) * g.HB * NT;
            int hb, a;
            task_slot(p, s, lp, int(cid) + i * int(ncl), hb, a);
            // the peers' h rows of this task land on xbar[xb]
            if (tid == 0) bar_expect(&s.xbar[xb], uint32_t(g.C - 1) * uint32_t(hrows * NT * 4));
            // gate/up of this warp's row groups over its quads
            bool got = ok;
            const int q0 = gu_q0(g, warp);
            for (int ri = 0; ri < g.RPW && got; ++ri) {
                const int rgl = gu_rgl(g, warp, ri);
                got = bar_wait(&s.gu_bar[b][rgl], ph);
                if (i == 0 && ri == 0) TRACEW(18 + warp);
                if (got) {
                    float ag[4] = {0.f, 0.f, 0.f, 0.f}, au[4] = {0.f, 0.f, 0.f, 0.f};
                    const uint8_t *gc = ring + size_t(b) * g.region + size_t(rgl) * g.gu_rg;
                    const uint8_t *uc = gc + (g.gu_c + g.gu_s);
                    for (int qi = 0; qi < g.QPW; ++qi) {
                        uint32_t B[4][8];
                        const uint4 *bq4 = bfx + size_t((q0 + qi) * 8) * (NT * 4) + lane;
#pragma unroll
                        for (int r4 = 0; r4 < 8; ++r4) {
                            const uint4 v = gl < NT ? bq4[r4 * (NT * 4)] : make_uint4(0u, 0u, 0u, 0u);
                            B[r4 >> 1][(r4 & 1) * 4 + 0] = v.x;
                            B[r4 >> 1][(r4 & 1) * 4 + 1] = v.y;
                            B[r4 >> 1][(r4 & 1) * 4 + 2] = v.z;
                            B[r4 >> 1][(r4 & 1) * 4 + 3] = v.w;
                        }
                        float xs[4][2];
#pragma unroll
                        for (int bq = 0; bq < 4; ++bq) {
                            xs[bq][0] = 2 * tl < T ? s.xs[4 * (q0 + qi) + bq][2 * tl] : 0.f;
                            xs[bq][1] = 2 * tl + 1 < T ? s.xs[4 * (q0 + qi) + bq][2 * tl + 1] : 0.f;
                        }
                        QuadRegs<FMT> qg, qu;
                        quad_smem<FMT>(gc, gc + g.gu_c, q0 + qi, lane, qg);
                        quad_smem<FMT>(uc, uc + g.gu_c, q0 + qi, lane, qu);
                        quad_pair_compute<FMT>(qg, qu, B, xs, ag, au);
                    }
                    float4 *dst = reinterpret_cast<float4 *>(red + (size_t(warp * g.RPW + ri) * 32 + lane) * 8);
                    dst[0] = make_float4(ag[0], ag[1], ag[2], ag[3]);
                    dst[1] = make_float4(au[0], au[1], au[2], au[3]);
                }
            }
            if (i == 0 && warp == 0) TRACEW(26);
            if (!got && ok && lane == 0) flag(p.status, MOE_DEV_TIMEOUT);
            ok = __syncthreads_and(ok && got) != 0;
            // the gate/up part of buffer b is free: copy ahead
            if (ok) issue_upto(nmine, i + 1, i);
            if (i == 0) TRACE(6);
            // h = silu(a) * u of this CTA's hidden rows (the WPR warps of a row group
            // summed in warp order), written to its rows of hs
            for (int e = tid; e < hrows * NT; e += kThreads) {
                const int r = e / NT, tok = e % NT;
                const int rgl = r >> 4, rr = r & 15;
                const int ln = 4 * (rr & 7) + (tok >> 1), ix = 2 * (rr >> 3) + (tok & 1);
                float A = 0.f, U = 0.f;
                for (int j = 0; j < g.WPR; ++j) {
                    const int w = g.WPR > 1 ? rgl * g.WPR + j : (rgl & 7);
                    const int ri = g.WPR > 1 ? 0 : (rgl >> 3);
                    const float *src = red + (size_t(w * g.RPW + ri) * 32 + ln) * 8 + ix;
                    A = j == 0 ? src[0] : A + src[0];
                    U = j == 0 ? src[4] : U + src[4];
                }
                const float h = (ok && tok < T) ? A / (1.0f + expf(-A)) * U : 0.f;
                too_big |= !(fabsf(h) <= 65504.f);
                hs[(int(rank) * hrows + r) * NT + tok] = h;
            }
            if (tid < NT) {  // gate of each token for this task
                float gw = 0.f;
                if (tid < T) {
                    if (a < 0) {
                        gw = 1.f;
                    } else {
                        for (int n = 0; n < s.act_cnt[a]; ++n) {
                            const int sp = s.act_beg[a] + n;
                            if (s.s_tok[sp] == tid) gw = s.w[tid][s.s_j[sp]];
                        }
                    }
                }
                s.gsel[tid] = gw;
            }
            __syncthreads();
            // push this CTA's h rows into every peer (16 bytes per store)
            {
                const int nv = hrows * NT / 4;
                const float4 *mine = reinterpret_cast<const float4 *>(hs + int(rank) * hrows * NT);
                for (int e = tid; e < nv * (g.C - 1); e += kThreads) {
                    const unsigned peer = (rank + 1 + unsigned(e / nv)) % unsigned(g.C);
                    const int v = e % nv;
                    st_async4(peer_addr(mine + v, peer), mine[v], peer_addr(&s.xbar[xb], peer));
                }
            }
            // the peers' h rows
            got = ok && bar_wait(&s.xbar[xb], xph);
            if (!got && ok && tid == 0) flag(p.status, MOE_DEV_TIMEOUT);
            ok = __syncthreads_and(got) != 0;
            if (i == 0) TRACE(7);
            // B fragments of h for the task's HB down columns (token columns < NT) and block sums
            const int nbh = g.HB / 64;
            for (int e = tid; e < nbh * 8 * 32; e += kThreads) {
                const int bq = e >> 8, rho = (e >> 5) & 7, ln = e & 31;
                const int gg = ln >> 2, tt = ln & 3;
                const int kk = 64 * bq + slot_k(rho, tt, 0);
                const float lo = gg < NT ? hs[kk * NT + gg] : 0.f, hi = gg < NT ? hs[(kk + 1) * NT + gg] : 0.f;
                const float sc = __int_as_float((127 - slot_exp<FMT>(bq, rho)) << 23);
                bfh[e] = pack_half2(lo * sc, hi * sc);
            }
            for (int job = warp; job < nbh * NT; job += kWarps) {
                const int bq = job / NT, n = job % NT;
                float v = hs[(64 * bq + lane) * NT + n] + hs[(64 * bq + 32 + lane) * NT + n];
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                if (lane == 0) s.hsb[bq][n] = v;
            }
            __syncthreads();
            // ---- down rows of this CTA over the task's columns (results staged in red)
            float *yst = red;
            got = ok && bar_wait(&s.dn_bar[b], ph);
            if (i == 0 && warp == 0) TRACEW(27);
            if (got) {
                const uint8_t *dcodes = ring + size_t(b) * g.region + g.gu_bytes;
                const uint8_t *dscales = dcodes + size_t(g.DR / 16) * g.dn_c;
                float xs[4][2];
#pragma unroll
                for (int bq = 0; bq < 4; ++bq) {
                    xs[bq][0] = bq < nbh && 2 * tl < T ? s.hsb[bq][2 * tl] : 0.f;
                    xs[bq][1] = bq < nbh && 2 * tl + 1 < T ? s.hsb[bq][2 * tl + 1] : 0.f;
                }
                auto stage = [&](int j, const float (&acc)[4]) {
                    const int rl = (warp * g.NDRW + j) * 16 + gl;  // row inside this CTA's DR rows
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        const int n = 2 * tl + (r & 1);
                        if (n < NT) yst[n * g.DR + rl + ((r & 2) ? 8 : 0)] = acc[r];
                    }
                };
                if constexpr (FMT == 2) {
                    uint32_t B[2][8];
#pragma unroll
                    for (int bq = 0; bq < 2; ++bq)
#pragma unroll
                        for (int rho = 0; rho < 8; ++rho) B[bq][rho] = bfh[(bq * 8 + rho) * 32 + lane];
                    const float xs2[2][2] = {{xs[0][0], xs[0][1]}, {xs[1][0], xs[1][1]}};
                    for (int j = 0; j < g.NDRW; j += 2) {  // NDRW is even (DR is a multiple of 256)
                        const int r0 = warp * g.NDRW + j;
                        const uint4 c0 = *reinterpret_cast<const uint4 *>(dcodes + size_t(r0) * g.dn_c + lane * 16);
                        const uint4 c1 =
                            *reinterpret_cast<const uint4 *>(dcodes + size_t(r0 + 1) * g.dn_c + lane * 16);
                        const uint4 s0 = *reinterpret_cast<const uint4 *>(dscales + size_t(r0) * g.dn_s + gl * 16);
                        const uint4 s1 =
                            *reinterpret_cast<const uint4 *>(dscales + size_t(r0 + 1) * g.dn_s + gl * 16);
                        float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
                        pair2_compute_q2(c0, s0, c1, s1, B, xs2, acc0, acc1);
                        stage(j, acc0);
                        stage(j + 1, acc1);
                    }
                } else {
                    uint32_t B[4][8];
#pragma unroll
                    for (int bq = 0; bq < 4; ++bq)
#pragma unroll
                        for (int rho = 0; rho < 8; ++rho) B[bq][rho] = bfh[(bq * 8 + rho) * 32 + lane];
                    for (int j = 0; j < g.NDRW; ++j) {
                        const int r0 = warp * g.NDRW + j;
                        QuadRegs<FMT> q;
                        quad_smem<FMT>(dcodes + size_t(r0) * g.dn_c, dscales + size_t(r0) * g.dn_s, 0, lane, q);
                        float acc[4] = {0.f, 0.f, 0.f, 0.f};
                        quad_compute_ilp<FMT>(q, B, xs, acc);
                        stage(j, acc);
                    }
                }
            }
            if (i == 0 && warp == 0) TRACEW(28);
            if (!got && ok && lane == 0) flag(p.status, MOE_DEV_TIMEOUT);
            ok = __syncthreads_and(ok && got) != 0;
            if (ok) issue_upto(nmine, i + 1, i + 1);  // the down part of buffer b is free
            if (i == 0) TRACE(8);
            // ---- gate-weighted vector atomics into y
            if (ok) {
                const int nv = T * (g.DR / 4);
                for (int e = tid; e < nv; e += kThreads) {
                    const int n = e / (g.DR / 4), r4 = e % (g.DR / 4);
                    const float gw = s.gsel[n];
                    if (gw != 0.f) {
                        const float4 v = *reinterpret_cast<const float4 *>(yst + n * g.DR + 4 * r4);
                        red_add4(lp.y + size_t(n) * d + int(rank) * g.DR + 4 * r4, gw * v.x, gw * v.y, gw * v.z,
                                 gw * v.w);
                    }
                }
            }
            __syncthreads();  // staging, h and fragments reused by the next task
            if (i == 0) TRACE(9);
        }
        seq += nmine;
        // copies issued for tasks that never ran (error paths) land before their buffers are reused
        if (gu_next > nmine || dn_next > nmine) {
            if (tid == 0)
                for (int i = nmine; i < max(gu_next, dn_next); ++i) {
                    const int b = (seq0 + i) % g.nbuf;
                    const uint32_t ph = uint32_t((seq0 + i) / g.nbuf) & 1u;
                    for (int r = 0; i < gu_next && r < g.GR; ++r) bar_wait(&s.gu_bar[b][r], ph);
                    if (i < dn_next) bar_wait(&s.dn_bar[b], ph);
                }
            __syncthreads();
            seq = seq0 + max(gu_next, dn_next);
        }
        if (ok && cta == G - 1) publish(p, s, l, T, k, E);
        // ------------------------------------------------ grid barrier: the layer is complete
        // (the next layer starts only once every contribution to this one is in y)
        if (l + 1 < p.L) {
            __syncthreads();  // this layer's tasks are done with the ring
            if (tid == 0) arrive_release(p.ctr);
            bar_target += unsigned(G);
            // the next layer's inputs (its own router rows and activations, which
            // this layer does not produce) into the ring while the barrier is pending
            const LayerPtrs np = layer_ptrs(p, l + 1);
            if (tid == 0 && nrows > 0) {
                bar_expect(&s.rt_bar, uint32_t(nrows) * uint32_t(d) * 4u);
                bulk_copy(rrows, np.Wr + size_t(rb) * d, uint32_t(nrows) * uint32_t(d) * 4u, &s.rt_bar);
            }
            {
                const uint4 *src = reinterpret_cast<const uint4 *>(np.x);
                uint4 *dst = reinterpret_cast<uint4 *>(sx);
                for (int i = tid; i < T * d / 8; i += kThreads) dst[i] = __ldg(src + i);
            }
            if (tid == 0) s.ok = wait_geq(p.ctr, bar_target, p.status);
            __syncthreads();
            ok = ok && s.ok;
        }
        TRACE(10);
    }

    if (too_big) flag(p.status, MOE_DEV_NONFINITE);
#ifdef MOE_DECODE_TRACE
    if (tid == 0) {
        unsigned long long t_;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));
        moe_decode_trace[blockIdx.x * 32 + 29] = t_;
        moe_decode_trace[blockIdx.x * 32 + 31] = clock64();
    }
#endif
    // no CTA leaves while a peer may still send into its shared memory
    asm volatile("barrier.cluster.arrive.relaxed.aligned;\nbarrier.cluster.wait.aligned;" ::: "memory");
    if (tid == 0) {
        __threadfence();
        s.last = atomicAdd(p.ctr + 1, 1u) == unsigned(G - 1);
    }
    __syncthreads();
    if (s.last && tid == 0) {  // every CTA is done with the counters: reset them for the next launch
        p.ctr[0] = 0u;
        __threadfence();
        p.ctr[1] = 0u;
        __threadfence();
    }
}

// ---------------------------------------------------------------- host side
size_t ws_align(size_t x) { return (x + 255) & ~size_t(255); }

// Cluster size for a format and hidden size: the hidden rows of a task (HB)
// and the down rows are split C ways. Q2 uses pairs of SMs (a task's weights
// on one CTA would be ~240 KB); Q3 (HB = 256) uses four.
int cluster_size(int fmt, int d, int cmax) {
    int c = fmt == 2 ? 2 : 4;
    c = std::min(c, cmax);
    while (c > 1 && d % (256 * c) != 0) c >>= 1;
    return c;
}
// (the launcher takes a larger cluster when a task of this one does not fit, e.g. Q3 with 8 tokens)

// Launch geometry and shared-memory layout for (fmt, T, d, f) with cluster size
// C, `avail` bytes of dynamic shared memory per CTA and G CTAs; false if it
// does not fit.
bool plan(int fmt, int T, int d, int f, int E, int G, int C, size_t avail, Geo &g) {
    g.C = C;
    g.HB = fmt == 2 ? 128 : 256;
    if (f % g.HB || d % 256 || g.HB % (16 * C)) return false;
    g.NHB = f / g.HB;
    g.GR = g.HB / C / 16;
    if (g.GR > 16) return false;
    g.RPW = g.GR > 8 ? g.GR / 8 : 1;
    g.WPR = g.GR < 8 ? 8 / g.GR : 1;
    g.NQ = d / 256;
    if (g.NQ % g.WPR) return false;
    g.QPW = g.NQ / g.WPR;
    g.DR = d / C;
    if (g.DR % 128) return false;
    g.NDRW = g.DR / 128;
    g.gu_c = uint32_t(g.NQ) * (fmt == 2 ? 1024u : 1536u);
    g.gu_s = uint32_t(g.NQ) * (fmt == 2 ? 256u : 128u);
    g.dn_c = fmt == 2 ? 512u : 1536u;
    g.dn_s = 128u;
    g.gu_rg = 2u * (g.gu_c + g.gu_s);
    g.gu_bytes = uint32_t(g.GR) * g.gu_rg;
    g.dn_bytes = uint32_t(g.DR / 16) * (g.dn_c + g.dn_s);
    if (g.gu_bytes % 128) return false;
    g.region = g.gu_bytes + g.dn_bytes;
    const int NTp = T <= 1 ? 1 : T <= 2 ? 2 : T <= 4 ? 4 : 8;
    g.red_bytes = uint32_t((std::max<size_t>(size_t(kWarps) * g.RPW * 32 * 8 * 4, size_t(NTp) * g.DR * 4) + 127) &
                           ~size_t(127));
    size_t off = 0;
    g.off_bfx = uint32_t(off);
    off += size_t(g.NQ) * 8 * NTp * 4 * 16;
    g.off_red = uint32_t(off);
    off += g.red_bytes;
    g.off_h = uint32_t(off);
    off += 2 * size_t(g.HB) * NTp * 4;
    g.off_bfh = uint32_t(off);
    off += size_t(g.HB / 64) * 1024;
    off = (off + 127) & ~size_t(127);
    g.off_ring = uint32_t(off);
    if (avail < off + g.region) return false;
    g.nbuf = int(std::min<size_t>(kMaxBuf, (avail - off) / g.region));
    const int rows = (E + G - 1) / G;
    const size_t router = size_t(rows) * d * 4 + size_t(T) * d * 2;  // router rows + x, staged in the ring
    size_t ring = size_t(g.nbuf) * g.region;
    if (ring < router) {
        if (off + router > avail) return false;
        ring = router;
    }
    g.total = uint32_t(off + ring);
    return true;
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// The down matrix of every slot of the pool as a 4D uint64 tensor [slot][row
// group][chunk][elements] for its codes and for its scales; a chunk is the
// codes (scales) of one row group over one block pair (Q2) or quad (Q3), and
// a box is one chunk of nrg consecutive row groups.
bool dn_maps(DecodeParams &p, int fmt, int d, int f, int nrg) {
    const MatGeom &m = p.down;
    const uint64_t nchunk = fmt == 2 ? uint64_t(m.NB / 2) : uint64_t(m.NB / 4);
    const uint64_t cb = fmt == 2 ? 512 : 1536;          // code bytes of a chunk
    const uint64_t sb = 128;                           // scale bytes of a chunk
    const uint64_t srow = fmt == 2 ? uint64_t(m.NB / 2) * 128 : uint64_t(m.NB / 2) * 64;  // scale bytes per row group
    const cuuint64_t cd[4] = {cb / 8, nchunk, cuuint64_t(d / 16), cuuint64_t(p.num_slots)};
    const cuuint64_t cs[3] = {cb, nchunk * cb, cuuint64_t(p.slot_bytes)};
    const cuuint32_t cbox[4] = {cuuint32_t(cb / 8), 1, cuuint32_t(nrg), 1};
    const cuuint64_t sd[4] = {sb / 8, nchunk, cuuint64_t(d / 16), cuuint64_t(p.num_slots)};
    const cuuint64_t ss[3] = {sb, srow, cuuint64_t(p.slot_bytes)};
    const cuuint32_t sbox[4] = {cuuint32_t(sb / 8), 1, cuuint32_t(nrg), 1};
    const cuuint32_t es[4] = {1, 1, 1, 1};
    (void)f;
    auto enc = [&](CUtensorMap *map, const uint8_t *base, const cuuint64_t *dims, const cuuint64_t *strides,
                   const cuuint32_t *box) {
        return g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT64, 4, const_cast<uint8_t *>(base), dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    };
    return enc(&p.dn_codes, p.pool + m.codes_off, cd, cs, cbox) &&
           enc(&p.dn_scales, p.pool + m.scales_off, sd, ss, sbox);
}

struct LaunchInfo {
    bool ready = false;
    int sms = 0;
    size_t avail = 0;   // dynamic shared memory a CTA can have
    int grid[9] = {};   // CTAs per launch for cluster size C (index C), 0 = not known yet
    bool coop = true;   // cooperative launches of clusters accepted
};
std::mutex g_mu;
LaunchInfo g_info[8][64];

template <int FMT, int NT>
moe_status launch(DecodeParams p, cudaStream_t stream) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    constexpr int ci = (FMT - 2) * 4 + (NT == 1 ? 0 : NT == 2 ? 1 : NT == 4 ? 2 : 3);
    auto kern = decode_layer_kernel<FMT, NT>;
    std::lock_guard<std::mutex> lock(g_mu);
    LaunchInfo &li = g_info[ci][dev];
    if (!li.ready) {
        int optin = 0, sms = 0;
        cudaFuncAttributes fa;
        if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess ||
            cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            cudaGetLastError();
            return MOE_ERR_CUDA;
        }
        const int av = optin - int(fa.sharedSizeBytes);
        if (av <= 0 || cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, av) != cudaSuccess) {
            cudaGetLastError();
            return MOE_ERR_CUDA;
        }
        li.sms = sms;
        li.avail = size_t(av);
        li.ready = true;
    }
    // the format's cluster size, doubled (up to 8) while a task does not fit in shared memory
    int C = cluster_size(FMT, p.d, 8), G = 0;
    for (;; C *= 2) {
        if (C > 8 || p.d % (256 * C) != 0) return MOE_ERR_UNSUPPORTED;
        if (li.grid[C] == 0) {  // co-resident clusters of C CTAs with the largest shared-memory use
            cudaLaunchConfig_t cfg = {};
            cudaLaunchAttribute at[1];
            at[0].id = cudaLaunchAttributeClusterDimension;
            at[0].val.clusterDim.x = unsigned(C);
            at[0].val.clusterDim.y = 1;
            at[0].val.clusterDim.z = 1;
            cfg.gridDim = dim3(unsigned(C * (li.sms / C)));
            cfg.blockDim = dim3(kThreads);
            cfg.dynamicSmemBytes = li.avail;
            cfg.attrs = at;
            cfg.numAttrs = 1;
            int ncl = 0;
            if (cudaOccupancyMaxActiveClusters(&ncl, kern, &cfg) != cudaSuccess || ncl < 1) {
                cudaGetLastError();
                return MOE_ERR_CUDA;
            }
            li.grid[C] = std::min(ncl * C, C * (li.sms / C));
        }
        G = li.grid[C];
        if (plan(FMT, p.T, p.d, p.f, p.E, G, C, li.avail, p.g)) break;
    }
    if (!g_encode) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn) {
            cudaGetLastError();
            return MOE_ERR_CUDA;
        }
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    if (!dn_maps(p, FMT, p.d, p.f, p.g.DR / 16)) return MOE_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = unsigned(C);
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    at[1].id = cudaLaunchAttributeCooperative;
    at[1].val.cooperative = 1;
    cfg.gridDim = dim3(unsigned(G));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = p.g.total;
    cfg.stream = stream;
    cfg.attrs = at;
    cfg.numAttrs = li.coop ? 2 : 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, p);
    if (e != cudaSuccess && li.coop) {
        // cooperative launches of clusters refused: the grid is sized to the co-resident
        // clusters and every grid-wide wait is bounded, so a plain cluster launch is used
        cudaGetLastError();
        li.coop = false;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, kern, p);
    }
    if (e != cudaSuccess) {
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

// Host-side checks and parameters shared by the one-layer and the stacked call.
moe_status setup(DecodeParams &p, const moe_qpool *W, int L, const int32_t *slot_of, const uint16_t *x,
                 const float *Wr, int T, int d, int f, int E, int k, int32_t miss_cap, moe_miss *miss, float *y,
                 void *ws, size_t ws_bytes) {
    if (!W || T < 0 || E <= 0 || k <= 0 || miss_cap < 0 || L < 1) return MOE_ERR_INVALID_ARG;
    if (W->fmt != 2 && W->fmt != 3) return MOE_ERR_INVALID_ARG;
    if (W->d != d || W->f != f) return MOE_ERR_INVALID_ARG;
    if (!dims_ok(d, f) || d > kMaxDimDec || f > kMaxFDec || T > kMaxTokDec || E > kMaxEDec || k > kMaxK || k > E)
        return MOE_ERR_UNSUPPORTED;
    if (int64_t(L) * E * d >= (int64_t(1) << 40)) return MOE_ERR_OVERFLOW;
    if (T == 0) return MOE_OK;
    if (!slot_of || !x || !Wr || !y) return MOE_ERR_INVALID_ARG;
    if (miss_cap > 0 && !miss) return MOE_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(x) % 16 || reinterpret_cast<uintptr_t>(Wr) % 16 ||
        reinterpret_cast<uintptr_t>(y) % 16)
        return MOE_ERR_INVALID_ARG;
    const ExpertGeom eg = expert_geom(W->fmt, d, f);
    if (!W->base || W->num_slots <= 0 || W->slot_bytes < int64_t(eg.bytes) || W->slot_bytes % 256 ||
        reinterpret_cast<uintptr_t>(W->base) % 256)
        return MOE_ERR_INVALID_ARG;
    if (!ws || ws_bytes < moe_layer_decode_workspace_bytes(T, k, f, E)) return MOE_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(ws) % 256) return MOE_ERR_INVALID_ARG;
    p = DecodeParams{};
    p.pool = static_cast<const uint8_t *>(W->base);
    p.slot_bytes = W->slot_bytes;
    p.num_slots = W->num_slots;
    p.L = L;
    p.slot_of = slot_of;
    p.x = x;
    p.Wr = Wr;
    p.T = T;
    p.d = d;
    p.f = f;
    p.E = E;
    p.k = k;
    p.miss = miss;
    p.miss_cap = miss_cap;
    p.y = y;
    unsigned char *w = static_cast<unsigned char *>(ws);
    p.ctr = reinterpret_cast<unsigned *>(w);
    p.logits = reinterpret_cast<float *>(w + 256);
    p.gate = eg.m[0];
    p.up = eg.m[1];
    p.down = eg.m[2];
    return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

MOE_API size_t moe_layer_decode_workspace_bytes(int T, int k, int f, int E) {
    if (T <= 0 || k <= 0 || f <= 0 || E <= 0) return 0;
    return 256 + ws_align(2 * size_t(kLogitCopies) * T * E * sizeof(float));
}

MOE_API size_t moe_stack_decode_workspace_bytes(int T, int k, int f, int E) {
    return moe_layer_decode_workspace_bytes(T, k, f, E);
}

// True for pinned host memory (mapped into the device's address space).
static bool in_host_memory(const void *ptr) {
    if (!ptr) return false;
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, ptr) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return a.type == cudaMemoryTypeHost;
}

MOE_API moe_status moe_layer_decode(const moe_qpool *W, const int32_t *slot_of, int32_t shared_slot, int32_t layer,
                                    const uint16_t *x, const float *Wr, const float *bias, int T, int d, int f, int E,
                                    int k, float *logits, int32_t *topk_idx, float *topk_w, int32_t *counts,
                                    int32_t *offsets, int32_t *sorted_tok, int32_t *sorted_j, int32_t *inv,
                                    int32_t *active, int32_t *slot_of_pair, moe_miss *miss, int32_t *miss_count,
                                    int32_t miss_cap, int32_t *expert_counts, float *y, void *ws, size_t ws_bytes,
                                    int32_t *dev_status, moe_stream_t stream) {
    DecodeParams p;
    const moe_status st = setup(p, W, 1, slot_of, x, Wr, T, d, f, E, k, miss_cap, miss, y, ws, ws_bytes);
    if (st != MOE_OK || T == 0) return st;
    if (shared_slot < 0 || shared_slot >= W->num_slots) return MOE_ERR_INVALID_ARG;
    p.shared_slot = nullptr;
    p.shared_slot0 = shared_slot;
    p.layer0 = layer;
    p.bias = bias;
    p.logits_out = logits;
    p.topk_idx = topk_idx;
    p.topk_w = topk_w;
    p.counts = counts;
    p.offsets = offsets;
    p.sorted_tok = sorted_tok;
    p.sorted_j = sorted_j;
    p.inv = inv;
    p.active = active;
    p.slot_of_pair = slot_of_pair;
    p.miss_count = miss_count;
    p.expert_counts = expert_counts;
    p.miss_host = in_host_memory(miss) || in_host_memory(miss_count);
    p.status = dev_status;
    return W->fmt == 2 ? launch_fmt<2>(p, as_cuda(stream)) : launch_fmt<3>(p, as_cuda(stream));
}

MOE_API moe_status moe_stack_decode(const moe_qpool *W, int L, const int32_t *slot_of, const int32_t *shared_slot,
                                    int32_t layer0, const uint16_t *x, const float *Wr, const float *bias, int T,
                                    int d, int f, int E, int k, int32_t *topk_idx, float *topk_w,
                                    int32_t *slot_of_pair, moe_miss *miss, int32_t *miss_count, int32_t miss_cap,
                                    int32_t *expert_counts, float *y, void *ws, size_t ws_bytes,
                                    int32_t *dev_status, moe_stream_t stream) {
    DecodeParams p;
    const moe_status st = setup(p, W, L, slot_of, x, Wr, T, d, f, E, k, miss_cap, miss, y, ws, ws_bytes);
    if (st != MOE_OK || T == 0) return st;
    if (!shared_slot) return MOE_ERR_INVALID_ARG;
    p.shared_slot = shared_slot;
    p.layer0 = layer0;
    p.bias = bias;
    p.topk_idx = topk_idx;
    p.topk_w = topk_w;
    p.slot_of_pair = slot_of_pair;
    p.miss_count = miss_count;
    p.expert_counts = expert_counts;
    p.miss_host = in_host_memory(miss) || in_host_memory(miss_count);
    p.status = dev_status;
    return W->fmt == 2 ? launch_fmt<2>(p, as_cuda(stream)) : launch_fmt<3>(p, as_cuda(stream));
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
