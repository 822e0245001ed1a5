// SwiGLU experts on packed 2-bit / 3-bit weights: weight-streaming kernels for
// small token counts per expert (decode, MTP verify batches).
//
// Each warp streams 16-row x 256-column tiles of codes with 16-byte coalesced
// loads and turns every 32-bit word straight into m16n8k16 fp16 A fragments:
// a code field at bit offset b of a half is the fp16 subnormal q*2^(b-24), so
// one AND yields a register and the products q*x are exact in the fp32
// accumulator. The activation fragment (B, up to 8 tokens) is pre-divided by
// 2^b per slot. Each 64-weight block gets a fresh accumulator; its scale and
// min are applied on the CUDA cores:  sum_k w_k x_k = s*sum_k q_k x_k + m*sum_k x_k
// (Q2) or s*sum_k q_k x_k - 4s*sum_k x_k (Q3), with the block sums of x
// computed once per token.
//
// The expert structure (10 routed of 512 plus a shared expert per token) is
// that of "个人开发者用 AI 十天写出 Strata 引擎，让 12GB 显存跑起 1250 亿参数的 Qwen 3.8
// Flash Next" (section "1250 亿参数，每个词只用得上 2%"); the SwiGLU form
// h = silu(Wg x) * (Wu x), y = Wd h and the Q2/Q3 formats are this library's.
#include <cuda_fp16.h>
#include <algorithm>
#include <math.h>
#include <mutex>

#include "common.cuh"
#include "layout.h"
#include "mma_q.cuh"

namespace moe {
namespace {

struct FfnParams {
    const uint8_t *pool;
    int64_t slot_bytes;
    int num_slots;
    const int32_t *slot_of;
    const uint16_t *x;
    int T, d, f, E, k;
    const int32_t *offsets, *sorted_tok, *sorted_j, *active;
    const float *topk_w;
    float *out;
    float *h;
    int32_t *status;
    MatGeom gate, up, down;
};

constexpr int kTokChunk = 8;

// Gate/up: CTA = (row group rg of f, active expert a); 8 warps split d in
// 256-column quads; writes h = silu(a) * u for the expert's tokens.
template <int FMT>
__global__ void __launch_bounds__(256) gateup_kernel(FfnParams p) {
    __shared__ float s_xs[kMaxDim / 64][kTokChunk];
    __shared__ float s_red[8][2][4][32];
    __shared__ int s_tok[kTokChunk];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int rg = blockIdx.x, a = blockIdx.y;
    if (a >= p.active[0]) return;
    const int e = p.active[1 + a];
    if (e < 0 || e >= p.E) {
        if (threadIdx.x == 0) flag(p.status, MOE_DEV_BAD_INDEX);
        return;
    }
    const int slot = p.slot_of[e];
    if (slot < 0) return;  // not resident: handled off the GPU
    if (slot >= p.num_slots) {
        if (threadIdx.x == 0) flag(p.status, MOE_DEV_BAD_SLOT);
        return;
    }
    const uint8_t *rec = p.pool + int64_t(slot) * p.slot_bytes;
    const int beg = p.offsets[e], cnt = p.offsets[e + 1] - beg;
    const int NB = p.d / 64, NQ = p.d / 256;
    bool too_big = false;
    for (int c0 = 0; c0 < cnt; c0 += kTokChunk) {
        const int nc = min(kTokChunk, cnt - c0);
        if (threadIdx.x < kTokChunk) s_tok[threadIdx.x] = threadIdx.x < nc ? p.sorted_tok[beg + c0 + threadIdx.x] : -1;
        __syncthreads();
        for (int i = threadIdx.x; i < NB * kTokChunk; i += blockDim.x) {
            const int b = i / kTokChunk, n = i % kTokChunk;
            float s = 0.f;
            if (n < nc) {
                const uint32_t *xr = reinterpret_cast<const uint32_t *>(p.x + int64_t(s_tok[n]) * p.d + 64 * b);
#pragma unroll 8
                for (int j = 0; j < 32; ++j) {
                    const uint32_t u = __ldg(xr + j);
                    s += bf16_lo(u) + bf16_hi(u);
                }
            }
            s_xs[b][n] = s;
        }
        __syncthreads();
        float ag[4] = {0.f, 0.f, 0.f, 0.f}, au[4] = {0.f, 0.f, 0.f, 0.f};
        const int tok = s_tok[g];
        const uint16_t *xrow = tok >= 0 ? p.x + int64_t(tok) * p.d : nullptr;
        for (int qd = warp; qd < NQ; qd += 8) {
            uint32_t B[4][8];
            build_b_global<FMT>(xrow, qd, t, B, too_big);
            float xs[4][2];
#pragma unroll
            for (int bq = 0; bq < 4; ++bq) {
                xs[bq][0] = s_xs[4 * qd + bq][2 * t];
                xs[bq][1] = s_xs[4 * qd + bq][2 * t + 1];
            }
            quad_tile<FMT>(rec, p.gate, rg, qd, lane, B, xs, ag);
            quad_tile<FMT>(rec, p.up, rg, qd, lane, B, xs, au);
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            s_red[warp][0][r][lane] = ag[r];
            s_red[warp][1][r][lane] = au[r];
        }
        __syncthreads();
        if (threadIdx.x < 128) {
            const int L = threadIdx.x >> 2, r = threadIdx.x & 3;
            float A = 0.f, U = 0.f;
#pragma unroll
            for (int w = 0; w < 8; ++w) {
                A += s_red[w][0][r][L];
                U += s_red[w][1][r][L];
            }
            const int row = (L >> 2) + ((r & 2) ? 8 : 0);
            const int n = 2 * (L & 3) + (r & 1);
            if (n < nc) p.h[int64_t(beg + c0 + n) * p.f + 16 * rg + row] = A / (1.0f + expf(-A)) * U;
        }
        __syncthreads();
    }
    if (too_big) flag(p.status, MOE_DEV_NONFINITE);
}

// Down: CTA = (4 row groups of d, active expert a); each warp one row group
// over all of f; writes y_perm rows or gate-weighted atomic adds into y.
template <int FMT>
__global__ void __launch_bounds__(128) down_kernel(FfnParams p) {
    __shared__ float s_hs[kMaxDim / 64][kTokChunk];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int rg = blockIdx.x * 4 + warp, a = blockIdx.y;
    if (a >= p.active[0]) return;
    const int e = p.active[1 + a];
    if (e < 0 || e >= p.E) return;
    const int slot = p.slot_of[e];
    if (slot < 0 || slot >= p.num_slots) return;
    const uint8_t *rec = p.pool + int64_t(slot) * p.slot_bytes;
    const int beg = p.offsets[e], cnt = p.offsets[e + 1] - beg;
    const int NB = p.f / 64, NQ = p.f / 256;
    bool too_big = false;
    for (int c0 = 0; c0 < cnt; c0 += kTokChunk) {
        const int nc = min(kTokChunk, cnt - c0);
        __syncthreads();
        for (int i = threadIdx.x; i < NB * kTokChunk; i += blockDim.x) {
            const int b = i / kTokChunk, n = i % kTokChunk;
            float s = 0.f;
            if (n < nc) {
                const float4 *hr = reinterpret_cast<const float4 *>(p.h + int64_t(beg + c0 + n) * p.f + 64 * b);
#pragma unroll 4
                for (int j = 0; j < 16; ++j) {
                    const float4 v = hr[j];
                    s += (v.x + v.y) + (v.z + v.w);
                }
            }
            s_hs[b][n] = s;
        }
        __syncthreads();
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        const float *hrow = g < nc ? p.h + int64_t(beg + c0 + g) * p.f : nullptr;
        for (int qd = 0; qd < NQ; ++qd) {
            uint32_t B[4][8];
            build_b_global<FMT>(hrow, qd, t, B, too_big);
            float xs[4][2];
#pragma unroll
            for (int bq = 0; bq < 4; ++bq) {
                xs[bq][0] = s_hs[4 * qd + bq][2 * t];
                xs[bq][1] = s_hs[4 * qd + bq][2 * t + 1];
            }
            quad_tile<FMT>(rec, p.down, rg, qd, lane, B, xs, acc);
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int n = 2 * t + (r & 1);
            if (n >= nc) continue;
            const int pos = beg + c0 + n;
            const int row = 16 * rg + g + ((r & 2) ? 8 : 0);
            if (p.topk_w) {
                const int tk = p.sorted_tok[pos], j = p.sorted_j[pos];
                atomicAdd(p.out + int64_t(tk) * p.d + row, p.topk_w[int64_t(tk) * p.k + j] * acc[r]);
            } else {
                p.out[int64_t(pos) * p.d + row] = acc[r];
            }
        }
    }
    if (too_big) flag(p.status, MOE_DEV_NONFINITE);
}

template <int FMT>
moe_status ffn_launch(const moe_qpool *W, const int32_t *slot_of, const uint16_t *x, int T, int d, int f, int E,
                      int k, const int32_t *offsets, const int32_t *sorted_tok, const int32_t *sorted_j,
                      const int32_t *active, const float *topk_w, float *out, void *ws, size_t ws_bytes,
                      int32_t *dev_status, moe_stream_t stream) {
    if (!W || T < 0 || E <= 0 || k <= 0) return MOE_ERR_INVALID_ARG;
    if (W->fmt != FMT || W->d != d || W->f != f) return MOE_ERR_INVALID_ARG;
    if (!dims_ok(d, f) || E > kMaxE || k > kMaxK) return MOE_ERR_UNSUPPORTED;
    if (int64_t(T) * k >= (int64_t(1) << 31)) return MOE_ERR_OVERFLOW;
    if (T == 0) return MOE_OK;
    if (!W->base || !slot_of || !x || !offsets || !sorted_tok || !sorted_j || !active || !out)
        return MOE_ERR_INVALID_ARG;
    const ExpertGeom eg = expert_geom(FMT, d, f);
    if (W->num_slots <= 0 || W->slot_bytes < int64_t(eg.bytes) || W->slot_bytes % 256 ||
        reinterpret_cast<uintptr_t>(W->base) % 256)
        return MOE_ERR_INVALID_ARG;
    if (!ws || ws_bytes < moe_expert_ffn_workspace_bytes(T, k, d, f)) return MOE_ERR_WORKSPACE;
    FfnParams p;
    p.pool = static_cast<const uint8_t *>(W->base);
    p.slot_bytes = W->slot_bytes;
    p.num_slots = W->num_slots;
    p.slot_of = slot_of;
    p.x = x;
    p.T = T;
    p.d = d;
    p.f = f;
    p.E = E;
    p.k = k;
    p.offsets = offsets;
    p.sorted_tok = sorted_tok;
    p.sorted_j = sorted_j;
    p.active = active;
    p.topk_w = topk_w;
    p.out = out;
    p.h = static_cast<float *>(ws);
    p.status = dev_status;
    p.gate = eg.m[0];
    p.up = eg.m[1];
    p.down = eg.m[2];
    cudaStream_t s = as_cuda(stream);
    if (int64_t(T) * k >= kTcMinPairs && E <= kTcMaxE)  // many tokens per expert: tensor-core GEMMs
        return tc05_ffn(FMT, W, slot_of, x, T, d, f, E, k, offsets, sorted_tok, sorted_j, active, topk_w, out, ws,
                        dev_status, s);
    const int na_max = int(std::min<int64_t>(E, int64_t(T) * k));
    gateup_kernel<FMT><<<dim3(f / 16, na_max), 256, 0, s>>>(p);
    down_kernel<FMT><<<dim3(d / 64, na_max), 128, 0, s>>>(p);
    return launch_status();
}

}  // namespace
}  // namespace moe

using namespace moe;

MOE_API size_t moe_expert_ffn_workspace_bytes(int T, int k, int d, int f) {
    if (T <= 0 || k <= 0 || f <= 0 || d <= 0) return 0;
    const size_t h32 = size_t(T) * size_t(k) * size_t(f) * sizeof(float);
    if (int64_t(T) * k < kTcMinPairs) return h32;  // only the weight-streaming path can run
    // the tensor-core path may run (it also needs the fp16 activation rows)
    const size_t tc = tc05_xperm_offset(T, k, f) + size_t(T) * size_t(k) * size_t(d) * 2;
    return std::max(h32, tc);
}

MOE_API moe_status moe_expert_ffn_q2(const moe_qpool *W, const int32_t *slot_of, const uint16_t *x, int T, int d,
                                     int f, int E, int k, const int32_t *offsets, const int32_t *sorted_tok,
                                     const int32_t *sorted_j, const int32_t *active, const float *topk_w, float *out,
                                     void *ws, size_t ws_bytes, int32_t *dev_status, moe_stream_t stream) {
    return ffn_launch<2>(W, slot_of, x, T, d, f, E, k, offsets, sorted_tok, sorted_j, active, topk_w, out, ws,
                         ws_bytes, dev_status, stream);
}

MOE_API moe_status moe_expert_ffn_q3(const moe_qpool *W, const int32_t *slot_of, const uint16_t *x, int T, int d,
                                     int f, int E, int k, const int32_t *offsets, const int32_t *sorted_tok,
                                     const int32_t *sorted_j, const int32_t *active, const float *topk_w, float *out,
                                     void *ws, size_t ws_bytes, int32_t *dev_status, moe_stream_t stream) {
    return ffn_launch<3>(W, slot_of, x, T, d, f, E, k, offsets, sorted_tok, sorted_j, active, topk_w, out, ws,
                         ws_bytes, dev_status, stream);
}

// ---------------------------------------------------------------------------
// moe_expert_ffn_q2_noalloc: the same kernels with their h scratch in a fixed
// array inside the library, for callers that cannot allocate device memory.
namespace moe {
namespace {
constexpr size_t kNoAllocBytes = size_t(4) << 20;  // 4 MiB: T*k*f floats of h
constexpr int kNoAllocMaxDevices = 64;
}  // namespace
}  // namespace moe

// One copy per GPU that loads the library, kept until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[moe::kNoAllocBytes];

namespace moe {
namespace {
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[kNoAllocMaxDevices] = {};
void *g_noalloc_ctx[kNoAllocMaxDevices] = {};  // driver context the address belongs to
using CtxGetCurrentFn = int (*)(void **);
CtxGetCurrentFn g_ctx_get_current = nullptr;

// Device address of g_noalloc_scratch on the current device, looked up once per
// device and driver context (host code only sees a host-side stand-in under
// that name; after a context is destroyed, its addresses are gone).
moe_status noalloc_scratch(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    if (dev < 0 || dev >= kNoAllocMaxDevices) return MOE_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_ctx_get_current) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &fn, 4000, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn) {
            cudaGetLastError();
            return MOE_ERR_CUDA;
        }
        g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(fn);
    }
    void *ctx = nullptr;
    if (g_ctx_get_current(&ctx) != 0) return MOE_ERR_CUDA;
    if (!ctx || !g_noalloc_ptr[dev] || g_noalloc_ctx[dev] != ctx) {
        // (the runtime makes the device's primary context current here if none was)
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return MOE_ERR_CUDA;
        }
        if (g_ctx_get_current(&ctx) != 0 || !ctx) return MOE_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
        g_noalloc_ctx[dev] = ctx;
    }
    *out = g_noalloc_ptr[dev];
    return MOE_OK;
}
}  // namespace
}  // namespace moe

MOE_API moe_status moe_expert_ffn_q2_noalloc(const moe_qpool *W, const int32_t *slot_of, const uint16_t *x, int T,
                                             int d, int f, int E, int k, const int32_t *offsets,
                                             const int32_t *sorted_tok, const int32_t *sorted_j,
                                             const int32_t *active, const float *topk_w, float *out,
                                             int32_t *dev_status, moe_stream_t stream) {
    if (T > 0 && k > 0 && f > 0 && moe_expert_ffn_workspace_bytes(T, k, d, f) > kNoAllocBytes) return MOE_ERR_WORKSPACE;
    void *ws = nullptr;
    if (T > 0) {
        const moe_status st = noalloc_scratch(&ws);
        if (st != MOE_OK) return st;
    }
    return ffn_launch<2>(W, slot_of, x, T, d, f, E, k, offsets, sorted_tok, sorted_j, active, topk_w, out, ws,
                         kNoAllocBytes, dev_status, stream);
}
