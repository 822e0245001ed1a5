// Router logits (fixed-order fp32) and top-k gates.
//
// Per token a router scores the layer's experts and the top 10 of 512 are used
// ("个人开发者用 AI 十天写出 Strata 引擎，让 12GB 显存跑起 1250 亿参数的 Qwen 3.8 Flash
// Next", section "1250 亿参数，每个词只用得上 2%"). The logit's fp32 value is defined
// by a fixed order of operations (see moe_route in moe.h) that a warp follows
// natively: lane l owns elements 128i+4l+j, accumulates them with fused
// multiply-adds chunk by chunk, and the butterfly of shuffles acc += shfl_xor(acc, o)
// for o = 16..1 is exactly the pairwise combination of the definition.
#include <math.h>

#include <mutex>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kTokTile = 8;      // tokens per warp
constexpr int kWarpsPerCta = 4;  // experts per CTA

// One warp = one expert x up to 8 tokens.
__global__ void __launch_bounds__(kWarpsPerCta * 32)
    router_logits_kernel(const uint16_t *__restrict__ x, const float *__restrict__ Wr, const float *__restrict__ bias,
                         int T, int d, int E, float *__restrict__ logits, int32_t *status) {
    const int lane = threadIdx.x & 31;
    const int e = blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
    if (e >= E) return;
    const int t0 = blockIdx.y * kTokTile;
    const int nt = min(kTokTile, T - t0);
    const float *w = Wr + size_t(e) * d + 4 * lane;
    const uint16_t *xb = x + size_t(t0) * d + 4 * lane;
    float acc[kTokTile];
#pragma unroll
    for (int tt = 0; tt < kTokTile; ++tt) acc[tt] = 0.0f;
    const int nchunk = d / 128;
#pragma unroll 4
    for (int i = 0; i < nchunk; ++i) {
        const float4 wv = __ldg(reinterpret_cast<const float4 *>(w + 128 * i));
#pragma unroll
        for (int tt = 0; tt < kTokTile; ++tt) {
            if (tt < nt) {
                const uint2 xv = __ldg(reinterpret_cast<const uint2 *>(xb + size_t(tt) * d + 128 * i));
                float a = acc[tt];
                a = __fmaf_rn(bf16_lo(xv.x), wv.x, a);
                a = __fmaf_rn(bf16_hi(xv.x), wv.y, a);
                a = __fmaf_rn(bf16_lo(xv.y), wv.z, a);
                a = __fmaf_rn(bf16_hi(xv.y), wv.w, a);
                acc[tt] = a;
            }
        }
    }
#pragma unroll
    for (int tt = 0; tt < kTokTile; ++tt) {
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) acc[tt] = __fadd_rn(acc[tt], __shfl_xor_sync(0xffffffffu, acc[tt], o));
    }
    if (lane == 0) {
        const float b = bias ? bias[e] : 0.0f;
        for (int tt = 0; tt < nt; ++tt) {
            float v = bias ? __fadd_rn(acc[tt], b) : acc[tt];
            if (!isfinite(v)) flag(status, MOE_DEV_NONFINITE);
            logits[size_t(t0 + tt) * E + e] = v;
        }
    }
}

// Many tokens, shared-memory staging: a CTA of 8 warps owns 32 tokens x 16
// experts (two CTAs per SM); every 128-element chunk of the tile (16 Wr rows fp32,
// 32 x rows bf16, 16 KiB) is brought into a ring of shared-memory stages by
// cp.async, and each warp computes 8 tokens x 8 experts from it with lane l holding
// the 64 partial sums of element class l (elements 128i+4l+j), two tokens per
// packed fp32 fma. Rows past T or E are clamped to the last row (valid memory,
// results not stored), so the inner loop has no bounds tests. The lane partials
// are combined by a reduce-scatter that adds exactly the pairs the butterfly adds
// (lane l and lane l^o, o = 16..1), each sum formed once.
constexpr int kRsTok = 32, kRsExp = 16, kRsThreads = 256, kRsStages = 4, kRsChunksPerSync = 2;
constexpr int kRsWBytes = kRsExp * 128 * 4, kRsXBytes = kRsTok * 128 * 2;
constexpr int kRsStageBytes = kRsWBytes + kRsXBytes;
constexpr int kRsSmem = kRsStages * kRsStageBytes;
constexpr int kWP = kRsExp * 32 / kRsThreads, kXP = kRsTok * 16 / kRsThreads;
static_assert(kWP * kRsThreads == kRsExp * 32 && kXP * kRsThreads == kRsTok * 16, "pieces");
constexpr int kWE = kRsExp / 8;  // expert groups of warps

__device__ __forceinline__ void rs_cp16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void rs_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void rs_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__global__ void __launch_bounds__(kRsThreads, 2)
    router_smem_kernel(const uint16_t *__restrict__ x, const float *__restrict__ Wr, const float *__restrict__ bias,
                       int T, int d, int E, float *__restrict__ logits, int32_t *status) {
    extern __shared__ __align__(128) uint8_t rs_smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int t0 = blockIdx.y * kRsTok, e0 = blockIdx.x * kRsExp;
    const uint32_t sbase = uint32_t(__cvta_generic_to_shared(rs_smem));
    // this thread's 16-byte pieces of a chunk: Wr pieces tid + n*256 (32 per row),
    // x pieces tid + n*256 (16 per row)
    const float *wsrc[kWP];
    uint32_t wdst[kWP];
    const uint16_t *xsrc[kXP];
    uint32_t xdst[kXP];
#pragma unroll
    for (int n = 0; n < kWP; ++n) {
        const int p = tid + n * kRsThreads, r = p >> 5, c = p & 31;
        wsrc[n] = Wr + size_t(min(e0 + r, E - 1)) * d + 4 * c;
        wdst[n] = r * 512 + c * 16;
    }
#pragma unroll
    for (int n = 0; n < kXP; ++n) {
        const int p = tid + n * kRsThreads, r = p >> 4, c = p & 15;
        xsrc[n] = x + size_t(min(t0 + r, T - 1)) * d + 8 * c;
        xdst[n] = kRsWBytes + r * 256 + c * 16;
    }
    const int nchunk = d / 128;
    auto load = [&](int chunk) {
        const uint32_t st = sbase + (chunk % kRsStages) * kRsStageBytes;
#pragma unroll
        for (int n = 0; n < kWP; ++n) rs_cp16(st + wdst[n], wsrc[n] + 128 * chunk);
#pragma unroll
        for (int n = 0; n < kXP; ++n) rs_cp16(st + xdst[n], xsrc[n] + 128 * chunk);
    };
    // chunks in flight ahead of the one computed; one barrier per kRsChunksPerSync chunks
    constexpr int kPre = kRsStages - kRsChunksPerSync;
#pragma unroll
    for (int c = 0; c < kPre; ++c) {
        if (c < nchunk) load(c);
        rs_commit();
    }
    const int wt = warp / kWE, we = warp % kWE;  // warp's 8-token and 8-expert group
    // acc[q][u]: logits of tokens 2q and 2q+1 with expert u, advanced together by
    // one packed fma per element (each half a single-rounding fp32 fma)
    float2 acc[4][8];
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int u = 0; u < 8; ++u) acc[q][u] = make_float2(0.f, 0.f);
    for (int i = 0; i < nchunk; ++i) {
        if (i % kRsChunksPerSync == 0) {
            rs_wait<kPre - kRsChunksPerSync>();
            __syncthreads();
#pragma unroll
            for (int c = 0; c < kRsChunksPerSync; ++c) {
                if (i + kPre + c < nchunk) load(i + kPre + c);
                rs_commit();
            }
        }
        const uint8_t *st = rs_smem + (i % kRsStages) * kRsStageBytes;
        const float4 *ws = reinterpret_cast<const float4 *>(st) + (we * 8) * 32 + lane;
        const uint2 *xs = reinterpret_cast<const uint2 *>(st + kRsWBytes) + (wt * 8) * 32 + lane;
        float2 X[4][4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint2 xa = xs[(2 * q) * 32], xb = xs[(2 * q + 1) * 32];
            X[q][0] = make_float2(bf16_lo(xa.x), bf16_lo(xb.x));
            X[q][1] = make_float2(bf16_hi(xa.x), bf16_hi(xb.x));
            X[q][2] = make_float2(bf16_lo(xa.y), bf16_lo(xb.y));
            X[q][3] = make_float2(bf16_hi(xa.y), bf16_hi(xb.y));
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const float4 wv = ws[u * 32];
            const float2 w0 = make_float2(wv.x, wv.x), w1 = make_float2(wv.y, wv.y);
            const float2 w2 = make_float2(wv.z, wv.z), w3 = make_float2(wv.w, wv.w);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float2 c = acc[q][u];
                c = __ffma2_rn(X[q][0], w0, c);
                c = __ffma2_rn(X[q][1], w1, c);
                c = __ffma2_rn(X[q][2], w2, c);
                c = __ffma2_rn(X[q][3], w3, c);
                acc[q][u] = c;
            }
        }
    }
    rs_wait<0>();
    // reduce-scatter over the 64 logits n = 8v + u: at offset o the lane with bit o
    // set keeps the upper half of its current values, its partner the lower half
    float r[64];
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            r[8 * (2 * q) + u] = acc[q][u].x;
            r[8 * (2 * q + 1) + u] = acc[q][u].y;
        }
#pragma unroll
    for (int lv = 0; lv < 5; ++lv) {
        const int o = 16 >> lv, m = 64 >> lv, hm = m >> 1;
        const bool up = lane & o;
#pragma unroll
        for (int j = 0; j < hm; ++j) {
            const float keep = up ? r[j + hm] : r[j];
            const float send = up ? r[j] : r[j + hm];
            r[j] = __fadd_rn(keep, __shfl_xor_sync(0xffffffffu, send, o));
        }
    }
    // lane l now holds logits n = 2l, 2l+1: token 8wt + (l >> 2), experts 8we + 2(l & 3) + {0,1}
    const int t = t0 + wt * 8 + (lane >> 2);
    const int e = e0 + we * 8 + 2 * (lane & 3);
    if (t < T) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            if (e + j < E) {
                const float v = bias ? __fadd_rn(r[j], bias[e + j]) : r[j];
                if (!isfinite(v)) flag(status, MOE_DEV_NONFINITE);
                logits[size_t(t) * E + e + j] = v;
            }
        }
    }
}

// (v1, i1) comes before (v2, i2): larger logit first, then lower id. NaN never wins.
__device__ __forceinline__ bool before(float v1, int i1, float v2, int i2) {
    return v1 > v2 || (v1 == v2 && i1 < i2);
}

// One warp per token: k rounds of warp-wide arg-max, then softmax over the k.
__global__ void topk_kernel(const float *__restrict__ logits, int T, int E, int k, int32_t *__restrict__ idx,
                            float *__restrict__ gate, int32_t *status) {
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    const float *row = logits + size_t(t) * E;
    uint32_t taken[kMaxE / 32 / 32];  // bit m of word m/32: candidate lane + 32*m taken
#pragma unroll
    for (int i = 0; i < kMaxE / 1024; ++i) taken[i] = 0;
    const int per_lane = (E + 31) / 32;
    bool saw_nan = false;
    int sel_id[kMaxK];
    float sel_v[kMaxK];
    for (int r = 0; r < k; ++r) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
        for (int m = 0; m < per_lane; ++m) {
            const int e = lane + 32 * m;
            if (e >= E) break;
            if ((taken[m >> 5] >> (m & 31)) & 1u) continue;
            const float v = row[e];
            if (v != v) {
                saw_nan = true;
                continue;
            }
            if (before(v, e, bv, bi)) {
                bv = v;
                bi = e;
            }
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (before(ov, oi, bv, bi)) {
                bv = ov;
                bi = oi;
            }
        }
        if (bi == 0x7fffffff) {  // only NaN left: no valid choice
            bi = 0;
            saw_nan = true;
        }
        if ((bi & 31) == lane) {
            const int m = bi >> 5;
            taken[m >> 5] |= 1u << (m & 31);
        }
        sel_id[r] = bi;
        sel_v[r] = bv;
    }
    if (saw_nan) flag(status, MOE_DEV_NONFINITE);
    if (lane == 0) {
        // selection order is by value; sort by id for the output
        for (int a = 1; a < k; ++a) {
            const int id = sel_id[a];
            const float v = sel_v[a];
            int b = a - 1;
            while (b >= 0 && sel_id[b] > id) {
                sel_id[b + 1] = sel_id[b];
                sel_v[b + 1] = sel_v[b];
                --b;
            }
            sel_id[b + 1] = id;
            sel_v[b + 1] = v;
        }
        float mx = -INFINITY;
        for (int a = 0; a < k; ++a) mx = fmaxf(mx, sel_v[a]);
        float z = 0.0f;
        float ex[kMaxK];
        for (int a = 0; a < k; ++a) {
            ex[a] = expf(sel_v[a] - mx);
            z += ex[a];
        }
        const float inv = 1.0f / z;
        for (int a = 0; a < k; ++a) {
            idx[size_t(t) * k + a] = sel_id[a];
            gate[size_t(t) * k + a] = ex[a] * inv;
        }
    }
}

// Order-preserving 32-bit key of an fp32 logit: larger logit -> larger key; +0
// and -0 share a key; 0 marks NaN (never above a number).
__device__ __forceinline__ uint32_t logit_key32(float v) {
    if (v != v) return 0u;
    if (v == 0.f) v = 0.f;
    const uint32_t u = __float_as_uint(v);
    const uint32_t k = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return k == 0u ? 1u : k;
}

// E <= 512: one warp per token with the token's logits in registers as 64-bit
// candidates (logit key << 32 | ~id: larger = larger logit, then lower id).
// Round r takes the warp-wide maximum (it is unique) into lane r; then the k
// selections are ranked by id and the gates computed exactly as topk_kernel
// does (maximum first, normaliser summed in ascending id, one reciprocal).
__global__ void __launch_bounds__(256)
    topk_reg_kernel(const float *__restrict__ logits, int T, int E, int k, int32_t *__restrict__ idx,
                    float *__restrict__ gate, int32_t *status) {
    constexpr int M = 512 / 32;
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    const float *row = logits + size_t(t) * E;
    uint64_t c[M];
    bool nan = false;
#pragma unroll
    for (int m = 0; m < M; ++m) {
        const int e = lane + 32 * m;
        if (e < E) {
            const float v = row[e];
            nan |= v != v;
            c[m] = (uint64_t(logit_key32(v)) << 32) | uint64_t(~uint32_t(e));
        } else {
            c[m] = 0ull;
        }
    }
    if (__any_sync(0xffffffffu, nan) && lane == 0) flag(status, MOE_DEV_NONFINITE);
    uint64_t mine = 0ull;
    for (int r = 0; r < k; ++r) {
        uint64_t mx = 0ull;
#pragma unroll
        for (int m = 0; m < M; ++m) mx = c[m] > mx ? c[m] : mx;
        const uint32_t hk = __reduce_max_sync(0xffffffffu, uint32_t(mx >> 32));
        const uint32_t lk = __reduce_max_sync(0xffffffffu, uint32_t(mx >> 32) == hk ? uint32_t(mx) : 0u);
        const uint64_t win = (uint64_t(hk) << 32) | lk;
        if (lane == r) mine = win;
        if (mx == win) {
#pragma unroll
            for (int m = 0; m < M; ++m)
                if (c[m] == win) c[m] = 0ull;
        }
    }
    // a round that found only NaN left takes expert 0 with logit -inf, as topk_kernel does
    const uint32_t key = uint32_t(mine >> 32);
    const int my_id = key ? int(~uint32_t(mine)) : 0;
    const float my_v = key ? __uint_as_float((key & 0x80000000u) ? (key ^ 0x80000000u) : ~key) : -INFINITY;
    const bool sel = lane < k;
    int rank = 0;  // position of this selection in ascending id order
    for (int q = 0; q < k; ++q) rank += __shfl_sync(0xffffffffu, my_id, q) < my_id;
    const float mx = __shfl_sync(0xffffffffu, my_v, 0);
    const float ex = sel ? expf(my_v - mx) : 0.f;
    float z = 0.0f;
    for (int a = 0; a < k; ++a) {
        const unsigned who = __ballot_sync(0xffffffffu, sel && rank == a);
        z += __shfl_sync(0xffffffffu, ex, __ffs(who) - 1);
    }
    const float inv = 1.0f / z;
    if (sel) {
        idx[size_t(t) * k + rank] = my_id;
        gate[size_t(t) * k + rank] = ex * inv;
    }
}

}  // namespace
}  // namespace moe

using namespace moe;

MOE_API moe_status moe_route(const uint16_t *x, const float *Wr, const float *bias, int T, int d, int E, int k,
                             float *logits, int32_t *topk_idx, float *topk_w, int32_t *dev_status,
                             moe_stream_t stream) {
    if (T < 0 || d <= 0 || E <= 0 || k <= 0) return MOE_ERR_INVALID_ARG;
    if (d % 128 || d > kMaxDim || E > kMaxE || k > kMaxK || k > E) return MOE_ERR_UNSUPPORTED;
    if (int64_t(T) * E >= (int64_t(1) << 31) || int64_t(T) * k >= (int64_t(1) << 31)) return MOE_ERR_OVERFLOW;
    if (T == 0) return MOE_OK;
    if (!x || !Wr || !logits || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(Wr)) & 15) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = as_cuda(stream);
    if (T >= 64) {
        // the kernel's shared memory (64 KiB) needs the opt-in, once per device
        static std::mutex mu;
        static bool ready[64] = {};
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
            cudaGetLastError();
            return MOE_ERR_CUDA;
        }
        {
            std::lock_guard<std::mutex> lock(mu);
            if (!ready[dev]) {
                if (cudaFuncSetAttribute(router_smem_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kRsSmem) !=
                    cudaSuccess) {
                    cudaGetLastError();
                    return MOE_ERR_CUDA;
                }
                ready[dev] = true;
            }
        }
        dim3 g((E + kRsExp - 1) / kRsExp, (T + kRsTok - 1) / kRsTok);
        router_smem_kernel<<<g, kRsThreads, kRsSmem, s>>>(x, Wr, bias, T, d, E, logits, dev_status);
    } else {
        dim3 g1((E + kWarpsPerCta - 1) / kWarpsPerCta, (T + kTokTile - 1) / kTokTile);
        router_logits_kernel<<<g1, kWarpsPerCta * 32, 0, s>>>(x, Wr, bias, T, d, E, logits, dev_status);
    }
    const int wpb = 8;
    if (E <= 512)
        topk_reg_kernel<<<(T + wpb - 1) / wpb, wpb * 32, 0, s>>>(logits, T, E, k, topk_idx, topk_w, dev_status);
    else
        topk_kernel<<<(T + wpb - 1) / wpb, wpb * 32, 0, s>>>(logits, T, E, k, topk_idx, topk_w, dev_status);
    return launch_status();
}
