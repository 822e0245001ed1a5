// SwiGLU experts for many tokens per expert (prefill): grouped GEMMs on the
// 5th-generation tensor cores (tcgen05, fp16 x fp16 -> fp32 in TMEM).
//
// Prompt chunks of up to 8192 tokens ("个人开发者用 AI 十天写出 Strata 引擎，让 12GB 显存跑起
// 1250 亿参数的 Qwen 3.8 Flash Next", section "等最久的，是它读完你的代码") route ~160 tokens
// to each of 512 experts, so each expert is a GEMM with the weights as M (128
// rows per tile) and the expert's tokens as N (up to 128 per tile, padded to 16).
//
// One persistent CTA per SM walks the (expert, M-tile, N-tile) list; warps are
// specialised:
//   producers (4 warps)  dequantise the packed Q2 codes of the tile's weight
//                        rows straight into 128-byte-swizzled fp16 shared memory
//                        (w = s*q + m, one fp16 rounding) and gather/convert the
//                        token rows (bf16 -> fp16, exact for normal values);
//   MMA (1 thread)       issues tcgen05.mma per 16-wide K step into a TMEM
//                        accumulator (double-buffered across tiles);
//   epilogue (4 warps)   drains TMEM: h = silu(g) * u (gate/up kernel), or
//                        y_e / gate-weighted atomics (down kernel).
// Stages hand over through mbarriers; every wait is bounded and sets
// MOE_DEV_TIMEOUT instead of hanging.
#include <cuda_fp16.h>
#include <math.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "layout.h"
#include "tc05.cuh"

namespace moe {
namespace {

constexpr int kProdWarps = 8;
constexpr int kProd = 32 * kProdWarps;  // producer threads (warps 0-7)
constexpr int kEpi = 128;               // epilogue threads (warps 8-11)
constexpr int kEpiWarp0 = kProdWarps;
constexpr int kMmaWarp = kProdWarps + 4;
constexpr int kTcThreads = kProd + kEpi + 32;  // + MMA warp (12)
constexpr int kTileN = 256;  // tokens per tile (MMA N, padded to 16)
constexpr int kSub = 16384;  // 128 rows x 64 cols fp16, SW128
constexpr int kSubB = 32768;  // 256 rows x 64 cols fp16, SW128
constexpr unsigned long long kTcWaitNs = 200ull * 1000 * 1000;
constexpr int kMaxActive = 2048;  // experts per call on this path (E <= 2048)

struct TcParams {
    const uint8_t *pool;
    int64_t slot_bytes;
    int num_slots;
    const int32_t *slot_of;
    const uint16_t *x;
    int T, d, f, E, k;
    const int32_t *offsets, *sorted_tok, *sorted_j, *active;
    const float *topk_w;
    float *out;
    __half *h;  // [T*k][f] fp16 hidden rows (sorted pair order)
    int32_t *status;
    MatGeom gate, up, down;
};

// Tile order: every full 256-token tile of every expert first, then the
// experts' last (partial) tiles from largest to smallest, so the long tiles
// start early and the short ones fill the end.
struct TcSmem {
    uint64_t full[4], empty[4], tfull[2], tempty[2];
    uint32_t tmem_base;
    int abort;
    int nfull_tiles;                 // full tiles (all M-tiles included)
    int nact;
    int full_prefix[kMaxActive + 1];  // full tiles before active expert a (x MT)
    uint16_t part_list[kMaxActive];   // active experts with a partial tile, largest first
    uint8_t bucket[kMaxActive];       // 16-token size class of each active expert's partial tile (0 = none)
    int tok[kTileN];                  // token ids of the producers' current tile
    int npart;
    int bucket_start[18];
    int bucket_run[18];
};

// Whole CTA: build the tile order; returns the tile count.
__device__ int build_schedule(const TcParams &p, TcSmem &s, int MT) {
    const int na = p.active[0];
    const int tid = threadIdx.x, nthr = blockDim.x;
    __shared__ int bucket_cnt[17];
    __shared__ int part[kTcThreads];
    if (tid < 17) bucket_cnt[tid] = 0;
    const int per = (na + nthr - 1) / nthr;
    const int a0 = tid * per;
    int local = 0;
    __syncthreads();
    for (int i = 0; i < per; ++i) {
        const int a = a0 + i;
        if (a < na) {
            const int e = p.active[1 + a];
            const bool ok = e >= 0 && e < p.E;
            const int sl = ok ? p.slot_of[e] : -1;
            const int n = (ok && sl >= 0 && sl < p.num_slots) ? p.offsets[e + 1] - p.offsets[e] : 0;
            s.full_prefix[a + 1] = MT * (n / kTileN);
            local += MT * (n / kTileN);
            const int rem = n % kTileN;
            s.bucket[a] = uint8_t(rem ? (rem + 15) >> 4 : 0);  // 1..16
            if (rem) atomicAdd(&bucket_cnt[(rem + 15) >> 4], 1);
        }
    }
    part[tid] = local;
    __syncthreads();
    if (tid == 0) {
        int run = 0;
        for (int i = 0; i < nthr; ++i) {
            const int v = part[i];
            part[i] = run;
            run += v;
        }
        s.full_prefix[0] = 0;
        s.nfull_tiles = run;
        int pos = 0;  // buckets from largest (16) down
        for (int bk = 16; bk >= 1; --bk) {
            s.bucket_start[bk] = pos;
            s.bucket_run[bk] = 0;
            pos += bucket_cnt[bk];
        }
        s.npart = pos;
        s.nact = na;
    }
    __syncthreads();
    int run = part[tid];
    for (int i = 0; i < per; ++i) {
        const int a = a0 + i;
        if (a < na) {
            run += s.full_prefix[a + 1];
            s.full_prefix[a + 1] = run;
        }
    }
    // Partial tiles: within a size class, ascending active index, so every CTA
    // derives the same order (one warp, 32 experts at a time).
    if (tid < 32) {
        for (int g0 = 0; g0 < na; g0 += 32) {
            const int a = g0 + tid;
            const int bk = a < na ? s.bucket[a] : 0;
            const unsigned peers = __match_any_sync(0xffffffffu, bk);
            const int rank = __popc(peers & ((1u << tid) - 1));
            if (bk) s.part_list[s.bucket_start[bk] + s.bucket_run[bk] + rank] = uint16_t(a);
            __syncwarp();
            if (bk && rank == 0) s.bucket_run[bk] += __popc(peers);
            __syncwarp();
        }
    }
    __syncthreads();
    return s.nfull_tiles + MT * s.npart;
}

struct TileInfo {
    int e, slot, beg, rows, mi;
};

__device__ __forceinline__ TileInfo tile_info(const TcParams &p, const TcSmem &s, int tau, int MT) {
    int a, ni, local;
    if (tau < s.nfull_tiles) {
        int lo = 0, hi = s.nact;  // last a with full_prefix[a] <= tau
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (s.full_prefix[mid] <= tau) lo = mid; else hi = mid;
        }
        a = lo;
        local = tau - s.full_prefix[a];
        ni = local / MT;
    } else {
        const int q = tau - s.nfull_tiles;
        a = s.part_list[q / MT];
        local = q;
        ni = -1;  // the partial tile
    }
    TileInfo t;
    t.e = p.active[1 + a];
    t.slot = p.slot_of[t.e];
    t.mi = local % MT;
    const int beg = p.offsets[t.e], n = p.offsets[t.e + 1] - beg;
    if (ni < 0) ni = n / kTileN;
    t.beg = beg + kTileN * ni;
    t.rows = min(kTileN, n - kTileN * ni);
    return t;
}

// Half of a 16-byte Q2 lane chunk: block bb (0/1) of the pair, rows g, g+8,
// plus that block's (s_g, s_g8, m_g, m_g8).
struct HalfQ2 {
    uint2 cw, sc;
};

__device__ __forceinline__ HalfQ2 load_half_q2(const uint8_t *rec, const MatGeom &m, int rg, int blk, int L) {
    HalfQ2 c;
    const int pair = blk >> 1, bb = blk & 1;
    c.cw = __ldg(reinterpret_cast<const uint2 *>(rec + q2_chunk_off(m, rg, pair, L) + 8 * bb));
    c.sc = __ldg(reinterpret_cast<const uint2 *>(rec + scale_off(m, 2, rg, pair, L >> 2) + 8 * bb));
    return c;
}

// Dequantise into a 128-row x 64-col SW128 sub-tile: w = s*q + m in fp16
// (q made exact in fp16 by the 1024-offset trick, then one fused multiply-add).
__device__ __forceinline__ void store_half_q2(const HalfQ2 &c, int rgl, int L, unsigned char *sub) {
    const int g = L >> 2, t = L & 3;
    const __half2 k1024 = __half2half2(__ushort_as_half(0x6400));
    const __half2 s01 = *reinterpret_cast<const __half2 *>(&c.sc.x);
    const __half2 m01 = *reinterpret_cast<const __half2 *>(&c.sc.y);
    // rows g and g+8 share (row & 7) = g, so their chunk order is the same
    unsigned char *row0 = sub + (2 * rgl) * 1024 + g * 128 + 4 * t;  // row 16rgl+g (8-row group 2rgl)
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const uint32_t w = r ? c.cw.y : c.cw.x;
        const __half2 s2 = r ? __high2half2(s01) : __low2half2(s01);
        const __half2 m2 = r ? __high2half2(m01) : __low2half2(m01);
        unsigned char *rowp = row0 + r * 1024;  // row g+8 is in the next 8-row group
#pragma unroll
        for (int rho = 0; rho < 8; ++rho) {
            const uint32_t qbits = ((w >> (2 * rho)) & 0x00030003u) | 0x64006400u;
            const __half2 q = __hsub2(*reinterpret_cast<const __half2 *>(&qbits), k1024);
            const __half2 wv = __hfma2(s2, q, m2);
            const int j = 2 * (rho >> 1) + (rho & 1);  // 16-byte chunk of the row
            *reinterpret_cast<__half2 *>(rowp + ((j ^ g) << 4)) = wv;
        }
    }
}

__device__ __forceinline__ void set_abort(TcSmem &s, int32_t *status) {
    if (atomicExch(&s.abort, 1) == 0) flag(status, MOE_DEV_TIMEOUT);
}

// Copy 8 fp16 (or 8 bf16 converted) values into a B sub-tile row chunk.
__device__ __forceinline__ uint4 bf16x8_to_f16x8(uint4 v) {
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const __half2 hh = __floats2half2_rn(bf16_lo(u[q]), bf16_hi(u[q]));
        o[q] = *reinterpret_cast<const uint32_t *>(&hh);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// -------------------------------------------------------------------- gate/up
// Stage (64 of K): A_gate 16 KB, A_up 16 KB, B (256 tokens) 32 KB. TMEM: D_g
// columns 0..255, D_u 256..511 (one accumulator pair; the epilogue is short).
constexpr int kGuStages = 3;
constexpr int kGuStageBytes = 2 * kSub + kSubB;

__global__ void __launch_bounds__(kTcThreads, 1) tc_gateup_q2_kernel(TcParams p) {
    extern __shared__ __align__(1024) unsigned char dyn_raw[];
    unsigned char *dyn =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(dyn_raw) + 1023) & ~uintptr_t(1023));
    __shared__ TcSmem s;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int MT = p.f / 128, KS = p.d / 64;
    if (tid == 0) {
        for (int i = 0; i < kGuStages; ++i) {
            tc::mbar_init(&s.full[i], kProd);
            tc::mbar_init(&s.empty[i], 1);
        }
        tc::mbar_init(&s.tfull[0], 1);
        tc::mbar_init(&s.tempty[0], kEpi);
        s.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kMmaWarp) tc::tmem_alloc(&s.tmem_base, 512);
    const int total = build_schedule(p, s, MT);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = s.tmem_base;

    if (warp < kProdWarps) {  // --------------------------------------- producers
        // Per stage a thread loads 2 weight half-chunks and 8 token-row chunks
        // (8 lanes per 128-byte row piece); loads of stage ks+1 are issued
        // before stage ks is written, so they overlap the MMAs.
        int it = 0;
        const int sub_row = lane >> 3, chunk = lane & 7;
        for (int tau = blockIdx.x; tau < total && !s.abort; tau += gridDim.x) {
            const TileInfo ti = tile_info(p, s, tau, MT);
            const uint8_t *rec = p.pool + int64_t(ti.slot) * p.slot_bytes;
            asm volatile("bar.sync 1, %0;" ::"r"(kProd));  // previous tile's token list no longer read
            for (int r = tid; r < kTileN; r += kProd) s.tok[r] = r < ti.rows ? p.sorted_tok[ti.beg + r] : -1;
            asm volatile("bar.sync 1, %0;" ::"r"(kProd));
            int rows_tok[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) rows_tok[j] = s.tok[32 * j + 4 * warp + sub_row];
            HalfQ2 ch[2], chn[2];
            uint4 xv[8], xvn[8];
            auto load_stage = [&](int ks, HalfQ2 (&c)[2], uint4 (&v)[8]) {
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const int cidx = tid + kProd * i;  // 2 matrices x 8 row groups x 32 lanes
                    c[i] = load_half_q2(rec, (cidx >> 8) ? p.up : p.gate, 8 * ti.mi + ((cidx >> 5) & 7), ks,
                                        cidx & 31);
                }
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    if (rows_tok[j] >= 0)
                        v[j] = __ldg(reinterpret_cast<const uint4 *>(p.x + int64_t(rows_tok[j]) * p.d + 64 * ks) +
                                     chunk);
            };
            load_stage(0, ch, xv);
            for (int ks = 0; ks < KS; ++ks, ++it) {
                const int st = it % kGuStages;
                const uint32_t ph = (it / kGuStages) & 1;
                if (ks + 1 < KS) load_stage(ks + 1, chn, xvn);
                if (!tc::mbar_wait(&s.empty[st], ph ^ 1, kTcWaitNs)) {
                    set_abort(s, p.status);
                    break;
                }
                unsigned char *stage = dyn + st * kGuStageBytes;
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const int cidx = tid + kProd * i;
                    store_half_q2(ch[i], (cidx >> 5) & 7, cidx & 31, stage + ((cidx >> 8) ? kSub : 0));
                }
                unsigned char *bsub = stage + 2 * kSub;
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    if (rows_tok[j] >= 0)
                        *reinterpret_cast<uint4 *>(bsub + tc::sw128_off(32 * j + 4 * warp + sub_row, chunk * 8)) =
                            bf16x8_to_f16x8(xv[j]);
                tc::fence_proxy_async();
                tc::mbar_arrive(&s.full[st]);
#pragma unroll
                for (int i = 0; i < 2; ++i) ch[i] = chn[i];
#pragma unroll
                for (int j = 0; j < 8; ++j) xv[j] = xvn[j];
            }
        }
    } else if (warp < kMmaWarp) {  // ---------------------------------- epilogue
        const int q = warp - kEpiWarp0;  // TMEM lane quadrant (warp % 4)
        int tcount = 0;
        bool too_big = false;
        for (int tau = blockIdx.x; tau < total && !s.abort; tau += gridDim.x, ++tcount) {
            const TileInfo ti = tile_info(p, s, tau, MT);
            if (!tc::mbar_wait(&s.tfull[0], tcount & 1, kTcWaitNs)) {
                set_abort(s, p.status);
                break;
            }
            tc::fence_after();
            const int frow = 128 * ti.mi + 32 * q + lane;
            const uint32_t tg = tmem + (uint32_t(32 * q) << 16);
            for (int c0 = 0; c0 < ti.rows; c0 += 16) {
                float g[16], u[16];
                tc::tmem_ld16(tg + c0, g);
                tc::tmem_ld16(tg + 256 + c0, u);
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    if (c0 + j < ti.rows) {
                        const float hv = g[j] / (1.0f + __expf(-g[j])) * u[j];
                        too_big |= !(fabsf(hv) <= 65504.f);
                        p.h[int64_t(ti.beg + c0 + j) * p.f + frow] = __float2half_rn(hv);
                    }
                }
            }
            tc::fence_before();
            tc::mbar_arrive(&s.tempty[0]);
        }
        if (too_big) flag(p.status, MOE_DEV_NONFINITE);
    } else if (lane == 0) {  // --------------------------------------------- MMA
        int it = 0, tcount = 0;
        for (int tau = blockIdx.x; tau < total && !s.abort; tau += gridDim.x, ++tcount) {
            const TileInfo ti = tile_info(p, s, tau, MT);
            const int npad = (ti.rows + 15) & ~15;
            const uint32_t idesc = tc::idesc_f16(128, npad);
            if (!tc::mbar_wait(&s.tempty[0], (tcount & 1) ^ 1, kTcWaitNs)) {
                set_abort(s, p.status);
                break;
            }
            tc::fence_after();
            const uint32_t dg = tmem, du = tmem + 256;
            for (int ks = 0; ks < KS; ++ks, ++it) {
                const int st = it % kGuStages;
                const uint32_t ph = (it / kGuStages) & 1;
                if (!tc::mbar_wait(&s.full[st], ph, kTcWaitNs)) {
                    set_abort(s, p.status);
                    break;
                }
                tc::fence_after();
                const uint32_t base = tc::smem_u32(dyn + st * kGuStageBytes);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t bd = tc::desc_sw128(base + 2 * kSub + 32 * kk);
                    const uint32_t acc = (ks | kk) ? 1u : 0u;
                    tc::mma_f16(dg, tc::desc_sw128(base + 32 * kk), bd, idesc, acc);
                    tc::mma_f16(du, tc::desc_sw128(base + kSub + 32 * kk), bd, idesc, acc);
                }
                tc::mma_commit(&s.empty[st]);
            }
            tc::mma_commit(&s.tfull[0]);
        }
    }
    tc::fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc::fence_after();
        tc::tmem_dealloc(tmem, 512);
    }
}

// ----------------------------------------------------------------------- down
// Stage (64 of K): A 16 KB + B (256 hidden rows) 32 KB. TMEM: two 256-column
// accumulators (the epilogue of one tile overlaps the MMAs of the next).
constexpr int kDnStages = 4;
constexpr int kDnStageBytes = kSub + kSubB;

__global__ void __launch_bounds__(kTcThreads, 1) tc_down_q2_kernel(TcParams p) {
    extern __shared__ __align__(1024) unsigned char dyn_raw[];
    unsigned char *dyn =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(dyn_raw) + 1023) & ~uintptr_t(1023));
    __shared__ TcSmem s;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int MT = p.d / 128, KS = p.f / 64;
    if (tid == 0) {
        for (int i = 0; i < kDnStages; ++i) {
            tc::mbar_init(&s.full[i], kProd);
            tc::mbar_init(&s.empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&s.tfull[i], 1);
            tc::mbar_init(&s.tempty[i], kEpi);
        }
        s.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kMmaWarp) tc::tmem_alloc(&s.tmem_base, 512);
    const int total = build_schedule(p, s, MT);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = s.tmem_base;

    if (warp < kProdWarps) {  // --------------------------------------- producers
        int it = 0;
        const int sub_row = lane >> 3, chunk = lane & 7;
        for (int tau = blockIdx.x; tau < total && !s.abort; tau += gridDim.x) {
            const TileInfo ti = tile_info(p, s, tau, MT);
            const uint8_t *rec = p.pool + int64_t(ti.slot) * p.slot_bytes;
            HalfQ2 ch, chn;
            uint4 hv[8], hvn[8];
            auto load_stage = [&](int ks, HalfQ2 &c, uint4 (&v)[8]) {
                c = load_half_q2(rec, p.down, 8 * ti.mi + (tid >> 5), ks, lane);  // 8 row groups x 32 lanes
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int r = 32 * j + 4 * warp + sub_row;
                    if (r < ti.rows)
                        v[j] = __ldcg(reinterpret_cast<const uint4 *>(p.h + int64_t(ti.beg + r) * p.f + 64 * ks) + chunk);
                }
            };
            load_stage(0, ch, hv);
            for (int ks = 0; ks < KS; ++ks, ++it) {
                const int st = it % kDnStages;
                const uint32_t ph = (it / kDnStages) & 1;
                if (ks + 1 < KS) load_stage(ks + 1, chn, hvn);
                if (!tc::mbar_wait(&s.empty[st], ph ^ 1, kTcWaitNs)) {
                    set_abort(s, p.status);
                    break;
                }
                unsigned char *stage = dyn + st * kDnStageBytes;
                store_half_q2(ch, tid >> 5, lane, stage);
                unsigned char *bsub = stage + kSub;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int r = 32 * j + 4 * warp + sub_row;
                    if (r < ti.rows) *reinterpret_cast<uint4 *>(bsub + tc::sw128_off(r, chunk * 8)) = hv[j];
                }
                tc::fence_proxy_async();
                tc::mbar_arrive(&s.full[st]);
                ch = chn;
#pragma unroll
                for (int j = 0; j < 8; ++j) hv[j] = hvn[j];
            }
        }
    } else if (warp < kMmaWarp) {  // ---------------------------------- epilogue
        const int q = warp - kEpiWarp0;
        int tcount = 0;
        for (int tau = blockIdx.x; tau < total && !s.abort; tau += gridDim.x, ++tcount) {
            const TileInfo ti = tile_info(p, s, tau, MT);
            const int b = tcount & 1;
            const uint32_t ph = (tcount >> 1) & 1;
            if (!tc::mbar_wait(&s.tfull[b], ph, kTcWaitNs)) {
                set_abort(s, p.status);
                break;
            }
            tc::fence_after();
            const int drow = 128 * ti.mi + 32 * q + lane;
            const uint32_t td = tmem + (uint32_t(32 * q) << 16) + uint32_t(b * 256);
            for (int c0 = 0; c0 < ti.rows; c0 += 16) {
                float v[16];
                tc::tmem_ld16(td + c0, v);
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    if (c0 + j < ti.rows) {
                        const int pos = ti.beg + c0 + j;
                        if (p.topk_w) {
                            const int tk = p.sorted_tok[pos], jj = p.sorted_j[pos];
                            atomicAdd(p.out + int64_t(tk) * p.d + drow, p.topk_w[int64_t(tk) * p.k + jj] * v[j]);
                        } else {
                            p.out[int64_t(pos) * p.d + drow] = v[j];
                        }
                    }
                }
            }
            tc::fence_before();
            tc::mbar_arrive(&s.tempty[b]);
        }
    } else if (lane == 0) {  // --------------------------------------------- MMA
        int it = 0, tcount = 0;
        for (int tau = blockIdx.x; tau < total && !s.abort; tau += gridDim.x, ++tcount) {
            const TileInfo ti = tile_info(p, s, tau, MT);
            const int npad = (ti.rows + 15) & ~15;
            const uint32_t idesc = tc::idesc_f16(128, npad);
            const int b = tcount & 1;
            const uint32_t phb = (tcount >> 1) & 1;
            if (!tc::mbar_wait(&s.tempty[b], phb ^ 1, kTcWaitNs)) {
                set_abort(s, p.status);
                break;
            }
            tc::fence_after();
            const uint32_t dd = tmem + uint32_t(b * 256);
            for (int ks = 0; ks < KS; ++ks, ++it) {
                const int st = it % kDnStages;
                const uint32_t ph = (it / kDnStages) & 1;
                if (!tc::mbar_wait(&s.full[st], ph, kTcWaitNs)) {
                    set_abort(s, p.status);
                    break;
                }
                tc::fence_after();
                const uint32_t base = tc::smem_u32(dyn + st * kDnStageBytes);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_f16(dd, tc::desc_sw128(base + 32 * kk), tc::desc_sw128(base + kSub + 32 * kk), idesc,
                                (ks | kk) ? 1u : 0u);
                tc::mma_commit(&s.empty[st]);
            }
            tc::mma_commit(&s.tfull[b]);
        }
    }
    tc::fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc::fence_after();
        tc::tmem_dealloc(tmem, 512);
    }
}

std::mutex g_tc_mu;
bool g_tc_ready[64] = {};
int g_tc_sms[64] = {};

constexpr size_t kGuSmem = size_t(kGuStages) * kGuStageBytes + 1024;
constexpr size_t kDnSmem = size_t(kDnStages) * kDnStageBytes + 1024;

}  // namespace

// Launch the two grouped GEMMs (Q2); h is fp16 [T*k][f] inside the caller's workspace.
moe_status tc05_ffn_q2(const moe_qpool *W, const int32_t *slot_of, const uint16_t *x, int T, int d, int f, int E, int k,
                       const int32_t *offsets, const int32_t *sorted_tok, const int32_t *sorted_j, const int32_t *active,
                       const float *topk_w, float *out, void *ws, int32_t *dev_status, cudaStream_t stream) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    {
        std::lock_guard<std::mutex> lock(g_tc_mu);
        if (!g_tc_ready[dev]) {
            if (cudaFuncSetAttribute(tc_gateup_q2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kGuSmem)) !=
                    cudaSuccess ||
                cudaFuncSetAttribute(tc_down_q2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kDnSmem)) !=
                    cudaSuccess ||
                cudaDeviceGetAttribute(&g_tc_sms[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
                cudaGetLastError();
                return MOE_ERR_CUDA;
            }
            g_tc_ready[dev] = true;
        }
    }
    const ExpertGeom eg = expert_geom(2, d, f);
    TcParams p;
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
    p.h = static_cast<__half *>(ws);
    p.status = dev_status;
    p.gate = eg.m[0];
    p.up = eg.m[1];
    p.down = eg.m[2];
    const int grid = g_tc_sms[dev];
    tc_gateup_q2_kernel<<<grid, kTcThreads, kGuSmem, stream>>>(p);
    tc_down_q2_kernel<<<grid, kTcThreads, kDnSmem, stream>>>(p);
    return launch_status();
}

}  // namespace moe
