// Tensor-core helpers shared by the expert FFN kernels: m16n8k16 fragments
// built straight from packed 2-bit / 3-bit codes (see layout.h).
//
// A code field at bit offset b of an fp16 half is the subnormal q*2^(b-24), so
// one AND of a packed word yields an A-fragment register and every product q*x
// is exact in the fp32 accumulator; the B fragment (activations) is divided by
// 2^b per slot. Each 64-weight block gets a fresh accumulator; its scale and
// min are applied on the CUDA cores: sum_k w_k x_k = s*sum_k q_k x_k + m*sum_k x_k
// (Q2) or s*sum_k q_k x_k - 4s*sum_k x_k (Q3).
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "common.cuh"
#include "layout.h"

namespace moe {

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
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// c = A * B  (m16n8k16 with a zero accumulator input: no zeroed registers needed)
__device__ __forceinline__ void mma16816_zc(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                            uint32_t b0, uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%10,%10,%10};"
        : "=f"(c[0]), "=f"(c[1]), "=f"(c[2]), "=f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
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

// Packed codes and scales of one 16-row x 256-column tile (rows 16rg..,
// columns 256qd..) as one lane holds them.
template <int FMT>
struct QuadRegs;
template <>
struct QuadRegs<2> {
    uint4 c0, c1, s0, s1;
};
template <>
struct QuadRegs<3> {
    uint32_t W[12];
    uint2 s0, s1;
};

template <int FMT>
__device__ __forceinline__ void quad_load(const uint8_t *rec, const MatGeom &m, int rg, int qd, int lane,
                                          QuadRegs<FMT> &q) {
    const int g = lane >> 2;
    if constexpr (FMT == 2) {
        q.c0 = ld_stream128(rec + q2_chunk_off(m, rg, 2 * qd, lane));
        q.c1 = ld_stream128(rec + q2_chunk_off(m, rg, 2 * qd + 1, lane));
        q.s0 = ld_stream128(rec + scale_off(m, 2, rg, 2 * qd, g));
        q.s1 = ld_stream128(rec + scale_off(m, 2, rg, 2 * qd + 1, g));
    } else {
#pragma unroll
        for (int s = 0; s < 3; ++s) {
            const uint4 v = ld_stream128(rec + q3_word_off(m, rg, qd, lane, 4 * s));
            q.W[4 * s + 0] = v.x;
            q.W[4 * s + 1] = v.y;
            q.W[4 * s + 2] = v.z;
            q.W[4 * s + 3] = v.w;
        }
        q.s0 = ld_stream64(rec + scale_off(m, 3, rg, 2 * qd, g));
        q.s1 = ld_stream64(rec + scale_off(m, 3, rg, 2 * qd + 1, g));
    }
}

// The tile against the B fragments of 8 tokens; accumulates rows g, g+8 x
// tokens 2t, 2t+1 into acc.
template <int FMT>
__device__ __forceinline__ void quad_compute(const QuadRegs<FMT> &q, const uint32_t (&B)[4][8],
                                             const float (&xs)[4][2], float (&acc)[4]) {
    if constexpr (FMT == 2) {
        const uint32_t wg[4] = {q.c0.x, q.c0.z, q.c1.x, q.c1.z};
        const uint32_t wg8[4] = {q.c0.y, q.c0.w, q.c1.y, q.c1.w};
        const uint32_t sc[4] = {q.s0.x, q.s0.z, q.s1.x, q.s1.z};
        const uint32_t mn[4] = {q.s0.y, q.s0.w, q.s1.y, q.s1.w};
#pragma unroll
        for (int bq = 0; bq < 4; ++bq) {
            float c[4];
            mma16816_zc(c, q2_reg(wg[bq], 0), q2_reg(wg8[bq], 0), q2_reg(wg[bq], 1), q2_reg(wg8[bq], 1), B[bq][0],
                        B[bq][1]);
#pragma unroll
            for (int i = 1; i < 4; ++i)
                mma16816(c, q2_reg(wg[bq], 2 * i), q2_reg(wg8[bq], 2 * i), q2_reg(wg[bq], 2 * i + 1),
                         q2_reg(wg8[bq], 2 * i + 1), B[bq][2 * i], B[bq][2 * i + 1]);
            block_epilogue<2>(c, sc[bq], mn[bq], xs[bq][0], xs[bq][1], acc);
        }
    } else {
        const uint32_t sc[4] = {q.s0.x, q.s0.y, q.s1.x, q.s1.y};
#pragma unroll
        for (int bq = 0; bq < 4; ++bq) {
            float c[4];
            mma16816_zc(c, q3_reg(q.W, 8 * bq, 0), q3_reg(q.W, 8 * bq, 1), q3_reg(q.W, 8 * bq + 1, 0),
                        q3_reg(q.W, 8 * bq + 1, 1), B[bq][0], B[bq][1]);
#pragma unroll
            for (int i = 1; i < 4; ++i) {
                const int u0 = 8 * bq + 2 * i, u1 = u0 + 1;
                mma16816(c, q3_reg(q.W, u0, 0), q3_reg(q.W, u0, 1), q3_reg(q.W, u1, 0), q3_reg(q.W, u1, 1),
                         B[bq][2 * i], B[bq][2 * i + 1]);
            }
            block_epilogue<3>(c, sc[bq], 0u, xs[bq][0], xs[bq][1], acc);
        }
    }
}

template <int FMT>
__device__ __forceinline__ void quad_tile(const uint8_t *rec, const MatGeom &m, int rg, int qd, int lane,
                                          const uint32_t (&B)[4][8], const float (&xs)[4][2], float (&acc)[4]) {
    QuadRegs<FMT> q;
    quad_load<FMT>(rec, m, rg, qd, lane, q);
    quad_compute<FMT>(q, B, xs, acc);
}

// B fragments of one 256-column quad for token row `src` (nullptr = zeros).
// Element (k, n=g) of slot rho of block bq, lane t: columns 256qd + 64bq +
// 16(rho/2) + 8(rho%2) + 2t + {0,1}, divided by 2^slot_exp.
template <int FMT, typename SrcT>
__device__ __forceinline__ void build_b_global(const SrcT *src, int qd, int t, uint32_t (&B)[4][8], bool &too_big) {
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


// B fragments of one quad from a generic (shared-memory or coherent global)
// pointer to bf16 activations; nullptr = zeros.
template <int FMT>
__device__ __forceinline__ void build_b_bf16(const uint16_t *src, int qd, int t, uint32_t (&B)[4][8]) {
#pragma unroll
    for (int bq = 0; bq < 4; ++bq)
#pragma unroll
        for (int rho = 0; rho < 8; ++rho) {
            float lo = 0.f, hi = 0.f;
            if (src) {
                const uint32_t u = *reinterpret_cast<const uint32_t *>(src + 256 * qd + 64 * bq + slot_k(rho, t, 0));
                lo = bf16_lo(u);
                hi = bf16_hi(u);
            }
            const float sc = __int_as_float((127 - slot_exp<FMT>(bq, rho)) << 23);
            B[bq][rho] = pack_half2(lo * sc, hi * sc);
        }
}

}  // namespace moe
