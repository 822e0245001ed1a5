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

__device__ __forceinline__ uint4 ld_stream128(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint2 ld_stream64(const void *p) {
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}

// c += A * B  (m16n8k16, fp16 inputs, fp32 accumulate)
__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

// Q2 fragment register rho of a word (fields at bit 2*rho / 2*rho+16).
__device__ __forceinline__ uint32_t q2_reg(uint32_t w, int rho) {
    return rho < 5 ? (w & (0x00030003u << (2 * rho))) : ((w >> 10) & (0x00030003u << (2 * (rho - 5))));
}

// Q3 fragment register of unit u, row r (see q3_place in layout.h).
__device__ __forceinline__ uint32_t q3_reg(const uint32_t (&W)[12], int u, int r) {
    if (u < 30) {
        const int wp = u / 5, kind = u % 5;
        switch (kind) {
            case 0: return r ? ((W[2 * wp] >> 9) & 0x00070007u) : (W[2 * wp] & 0x00070007u);
            case 1: return r ? ((W[2 * wp] >> 9) & 0x00380038u) : (W[2 * wp] & 0x00380038u);
            case 2: return r ? ((W[2 * wp + 1] >> 9) & 0x00070007u) : (W[2 * wp + 1] & 0x00070007u);
            case 3: return r ? ((W[2 * wp + 1] >> 9) & 0x00380038u) : (W[2 * wp + 1] & 0x00380038u);
            default: return W[2 * wp + r] & 0x01C001C0u;
        }
    }
    const int b = 6 * (u - 30) + 3 * r;
    return ((W[b] >> 15) & 0x00010001u) | ((W[b + 1] >> 14) & 0x00020002u) | ((W[b + 2] >> 13) & 0x00040004u);
}

template <int FMT>
__device__ __forceinline__ int slot_exp(int bq, int rho) {
    return FMT == 2 ? q2_exp(rho) : q3_exp(8 * bq + rho);
}

// Block epilogue: acc += s*2^24 * c + m' * xsum.
template <int FMT>
__device__ __forceinline__ void block_epilogue(const float (&c)[4], uint32_t scale2, uint32_t min2, float xs0,
                                               float xs1, float (&acc)[4]) {
    const float2 sf = __half22float2(*reinterpret_cast<const __half2 *>(&scale2));
    const float S0 = sf.x * 16777216.0f, S1 = sf.y * 16777216.0f;
    float M0, M1;
    if (FMT == 2) {
        const float2 mf = __half22float2(*reinterpret_cast<const __half2 *>(&min2));
        M0 = mf.x;
        M1 = mf.y;
    } else {
        M0 = -4.0f * sf.x;
        M1 = -4.0f * sf.y;
    }
    acc[0] = fmaf(S0, c[0], fmaf(M0, xs0, acc[0]));
    acc[1] = fmaf(S0, c[1], fmaf(M0, xs1, acc[1]));
    acc[2] = fmaf(S1, c[2], fmaf(M1, xs0, acc[2]));
    acc[3] = fmaf(S1, c[3], fmaf(M1, xs1, acc[3]));
}

// One 16-row x 256-column tile (rows 16rg.., quad qd) of matrix m against the
// B fragments of 8 tokens; accumulates rows g, g+8 x tokens 2t, 2t+1 into acc.
template <int FMT>
__device__ __forceinline__ void quad_tile(const uint8_t *rec, const MatGeom &m, int rg, int qd, int lane,
                                          const uint32_t (&B)[4][8], const float (&xs)[4][2], float (&acc)[4]) {
    const int g = lane >> 2;
    if (FMT == 2) {
        const uint4 c0 = ld_stream128(rec + q2_chunk_off(m, rg, 2 * qd, lane));
        const uint4 c1 = ld_stream128(rec + q2_chunk_off(m, rg, 2 * qd + 1, lane));
        const uint4 s0 = ld_stream128(rec + scale_off(m, 2, rg, 2 * qd, g));
        const uint4 s1 = ld_stream128(rec + scale_off(m, 2, rg, 2 * qd + 1, g));
        const uint32_t wg[4] = {c0.x, c0.z, c1.x, c1.z};
        const uint32_t wg8[4] = {c0.y, c0.w, c1.y, c1.w};
        const uint32_t sc[4] = {s0.x, s0.z, s1.x, s1.z};
        const uint32_t mn[4] = {s0.y, s0.w, s1.y, s1.w};
#pragma unroll
        for (int bq = 0; bq < 4; ++bq) {
            float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int i = 0; i < 4; ++i)
                mma16816(c, q2_reg(wg[bq], 2 * i), q2_reg(wg8[bq], 2 * i), q2_reg(wg[bq], 2 * i + 1),
                         q2_reg(wg8[bq], 2 * i + 1), B[bq][2 * i], B[bq][2 * i + 1]);
            block_epilogue<2>(c, sc[bq], mn[bq], xs[bq][0], xs[bq][1], acc);
        }
    } else {
        uint32_t W[12];
#pragma unroll
        for (int s = 0; s < 3; ++s) {
            const uint4 v = ld_stream128(rec + q3_word_off(m, rg, qd, lane, 4 * s));
            W[4 * s + 0] = v.x;
            W[4 * s + 1] = v.y;
            W[4 * s + 2] = v.z;
            W[4 * s + 3] = v.w;
        }
        const uint2 s0 = ld_stream64(rec + scale_off(m, 3, rg, 2 * qd, g));
        const uint2 s1 = ld_stream64(rec + scale_off(m, 3, rg, 2 * qd + 1, g));
        const uint32_t sc[4] = {s0.x, s0.y, s1.x, s1.y};
#pragma unroll
        for (int bq = 0; bq < 4; ++bq) {
            float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int u0 = 8 * bq + 2 * i, u1 = u0 + 1;
                mma16816(c, q3_reg(W, u0, 0), q3_reg(W, u0, 1), q3_reg(W, u1, 0), q3_reg(W, u1, 1), B[bq][2 * i],
                         B[bq][2 * i + 1]);
            }
            block_epilogue<3>(c, sc[bq], 0u, xs[bq][0], xs[bq][1], acc);
        }
    }
}

// B fragments of one 256-column quad for token row `src` (nullptr = zeros).
// Element (k, n=g) of slot rho of block bq, lane t: columns 256qd + 64bq +
// 16(rho/2) + 8(rho%2) + 2t + {0,1}, divided by 2^slot_exp.
template <int FMT, typename SrcT>
__device__ __forceinline__ void build_b(const SrcT *src, int qd, int t, uint32_t (&B)[4][8], bool &too_big) {
#pragma unroll
    for (int bq = 0; bq < 4; ++bq)
#pragma unroll
        for (int rho = 0; rho < 8; ++rho) {
            float lo = 0.f, hi = 0.f;
            if (src) {
                const int kk = 256 * qd + 64 * bq + slot_k(rho, t, 0);
                if constexpr (sizeof(SrcT) == 2) {
                    const uint32_t u = __ldg(reinterpret_cast<const uint32_t *>(src + kk));
                    lo = bf16_lo(u);
                    hi = bf16_hi(u);
                } else {
                    const float2 v = __ldg(reinterpret_cast<const float2 *>(src + kk));
                    lo = v.x;
                    hi = v.y;
                }
                too_big |= !(fabsf(lo) <= 65504.f) || !(fabsf(hi) <= 65504.f);
            }
            const float sc = __int_as_float((127 - slot_exp<FMT>(bq, rho)) << 23);  // 2^-exp
            B[bq][rho] = pack_half2(lo * sc, hi * sc);
        }
}

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
            build_b<FMT>(xrow, qd, t, B, too_big);
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
            build_b<FMT>(hrow, qd, t, B, too_big);
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
    if (!ws || ws_bytes < moe_expert_ffn_workspace_bytes(T, k, f)) return MOE_ERR_WORKSPACE;
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
    const int na_max = int(std::min<int64_t>(E, int64_t(T) * k));
    cudaStream_t s = as_cuda(stream);
    gateup_kernel<FMT><<<dim3(f / 16, na_max), 256, 0, s>>>(p);
    down_kernel<FMT><<<dim3(d / 64, na_max), 128, 0, s>>>(p);
    return launch_status();
}

}  // namespace
}  // namespace moe

using namespace moe;

MOE_API size_t moe_expert_ffn_workspace_bytes(int T, int k, int f) {
    if (T <= 0 || k <= 0 || f <= 0) return 0;
    return size_t(T) * size_t(k) * size_t(f) * sizeof(float);
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

// Device address of g_noalloc_scratch on the current device, looked up once per
// device (host code only sees a host-side stand-in under that name).
moe_status noalloc_scratch(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    if (dev < 0 || dev >= kNoAllocMaxDevices) return MOE_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return MOE_ERR_CUDA;
        }
        g_noalloc_ptr[dev] = p;
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
    if (T > 0 && k > 0 && f > 0 && moe_expert_ffn_workspace_bytes(T, k, f) > kNoAllocBytes) return MOE_ERR_WORKSPACE;
    void *ws = nullptr;
    if (T > 0) {
        const moe_status st = noalloc_scratch(&ws);
        if (st != MOE_OK) return st;
    }
    return ffn_launch<2>(W, slot_of, x, T, d, f, E, k, offsets, sorted_tok, sorted_j, active, topk_w, out, ws,
                         kNoAllocBytes, dev_status, stream);
}
