// SwiGLU experts for many tokens per expert (prefill): grouped GEMMs on the
// 5th-generation tensor cores (tcgen05, fp16 x fp16 -> fp32 in TMEM).
//
// Prompt chunks of up to 8192 tokens ("个人开发者用 AI 十天写出 Strata 引擎，让 12GB 显存跑起
// 1250 亿参数的 Qwen 3.8 Flash Next", section "等最久的，是它读完你的代码") route ~160 tokens
// to each of 512 experts, so each expert is a GEMM with the weights as M (128
// rows per tile) and the expert's tokens as N (up to 256 per tile, padded to 16).
//
// One persistent CTA per SM walks the (expert, M-tile, N-tile) list; warps are
// specialised:
//   producers (8 warps)  copy each K stage's token rows (fp16) into
//                        128-byte-swizzled shared memory and the stage's packed
//                        Q2 codes and scales into a staging area, both with
//                        asynchronous cp.async copies issued two or three stages
//                        ahead; when a stage has landed they dequantise its codes
//                        into the fp16 A tile (w = s*q + m, one fp16 rounding);
//                        the next tile's weights are prefetched into L2;
//   MMA (1 thread)       issues tcgen05.mma per 16-wide K step into a TMEM
//                        accumulator;
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
constexpr int kRawMat = kProd * 16;  // packed codes + scales of one matrix, one stage
constexpr unsigned long long kTcWaitNs = 200ull * 1000 * 1000;
constexpr int kMaxActive = kTcMaxE;  // experts per call on this path

struct TcParams {
    const uint8_t *pool;
    int64_t slot_bytes;
    int num_slots;
    const int32_t *slot_of;
    const __half *x16;  // [T][d] fp16 copy of the activations
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
    int npart;
    int bucket_start[18];
    int bucket_run[18];
};

// Whole CTA: build the tile order; returns the tile count. scratch holds
// blockDim.x ints (the stage buffers, not yet in use).
__device__ int build_schedule(const TcParams &p, TcSmem &s, int MT, int *part) {
    const int na = p.active[0];
    const int tid = threadIdx.x, nthr = blockDim.x;
    __shared__ int bucket_cnt[17];
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

// The packed codes (8 B) and scale entry (8 B) of one block of one lane chunk:
// block bb of the pair, rows g and g+8, {s(g), s(g+8), m(g), m(g+8)}.
struct HalfQ2 {
    uint2 cw, sc;
};

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

// Ask the L2 for the weight rows of tile tau (codes and scales of each of the
// NMAT matrices, one contiguous range each) and, for the down GEMM, the hidden
// rows of the tile.
template <int NMAT, bool GATHER>
__device__ __forceinline__ void prefetch_tile(const TcParams &p, const TcSmem &s, int tau, int MT,
                                              const MatGeom *const *mats, int K) {
    const TileInfo t = tile_info(p, s, tau, MT);
    const uint8_t *rec = p.pool + int64_t(t.slot) * p.slot_bytes;
    const int npair = K / 128;
#pragma unroll
    for (int i = 0; i < NMAT; ++i) {
        const MatGeom &m = *mats[i];
        tc::prefetch_l2(rec + q2_chunk_off(m, 8 * t.mi, 0, 0), uint32_t(8 * npair * 512));
        tc::prefetch_l2(rec + scale_off(m, 2, 8 * t.mi, 0, 0), uint32_t(8 * npair * 128));
    }
    if (!GATHER && t.rows > 0) tc::prefetch_l2(p.h + int64_t(t.beg) * p.f, uint32_t(t.rows) * uint32_t(p.f) * 2u);
}

// Producer warps. Stage it lives in slot it % S: NMAT fp16 A sub-tiles, the B
// sub-tile (256 rows), and a staging area for the packed A bytes. A stage is
// issued L = S-1 stages ahead (wait until the MMA released the slot, then
// cp.async of B rows and packed A bytes, one commit group per stage and
// thread) and finished when its group has landed (dequantise the thread's own
// packed bytes into A, fence for the tensor core, arrive on full[slot]).
// GATHER: B row r is the fp16 activation row of token sorted_tok[beg + r]
// (K = d); otherwise the hidden row beg + r (K = f).
template <int NMAT, int S, bool GATHER>
__device__ __forceinline__ void produce(const TcParams &p, TcSmem &s, unsigned char *dyn, int total, int MT, int KS,
                        const MatGeom *const *mats) {
    constexpr int L = S - 1;
    constexpr int kStageBytes = NMAT * kSub + kSubB;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int sub_row = lane >> 3, chunk = lane & 7;
    const int K = GATHER ? p.d : p.f;
    const int mine = blockIdx.x < total ? (total - int(blockIdx.x) + int(gridDim.x) - 1) / int(gridDim.x) : 0;
    const int nstages = mine * KS;
    unsigned char *raw_base = dyn + S * kStageBytes;

    // issue cursor
    int i_tau = blockIdx.x, i_ks = 0;
    const uint8_t *i_rec = nullptr;
    int i_mi = 0;
    const __half *brow[8];
    auto enter_tile = [&]() {
        const TileInfo t = tile_info(p, s, i_tau, MT);
        i_rec = p.pool + int64_t(t.slot) * p.slot_bytes;
        i_mi = t.mi;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int r = 32 * j + 4 * warp + sub_row;
            brow[j] = nullptr;
            if (r < t.rows) {
                const int64_t row = GATHER ? int64_t(p.sorted_tok[t.beg + r]) : int64_t(t.beg + r);
                brow[j] = (GATHER ? p.x16 : p.h) + row * K + 8 * chunk;
            }
        }
        if (tid == 0 && i_tau + int(gridDim.x) < total)
            prefetch_tile<NMAT, GATHER>(p, s, i_tau + gridDim.x, MT, mats, K);
    };
    if (mine > 0) enter_tile();

    auto issue = [&](int it) -> bool {
        const int st = it % S;
        if (!tc::mbar_wait(&s.empty[st], ((it / S) & 1) ^ 1, kTcWaitNs)) return false;
        unsigned char *stage = dyn + st * kStageBytes;
        unsigned char *bsub = stage + NMAT * kSub;
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (brow[j])
                tc::cp_async16(bsub + tc::sw128_off(32 * j + 4 * warp + sub_row, chunk * 8), brow[j] + 64 * i_ks);
        unsigned char *raw = raw_base + st * (NMAT * kRawMat) + tid * 16;
        const int pair = i_ks >> 1, bb = i_ks & 1;
#pragma unroll
        for (int i = 0; i < NMAT; ++i) {
            const MatGeom &m = *mats[i];
            tc::cp_async8(raw + i * kRawMat, i_rec + q2_chunk_off(m, 8 * i_mi + warp, pair, lane) + 8 * bb);
            tc::cp_async8(raw + i * kRawMat + 8, i_rec + scale_off(m, 2, 8 * i_mi + warp, pair, lane >> 2) + 8 * bb);
        }
        if (++i_ks == KS) {
            i_ks = 0;
            i_tau += gridDim.x;
            if (i_tau < total) enter_tile();
        }
        return true;
    };

    bool ok = true;
#pragma unroll 1
    for (int q = 0; q < L; ++q) {
        if (ok && q < nstages) ok = issue(q);
        tc::cp_async_commit();
    }
#pragma unroll 1
    for (int it = 0; it < nstages && ok; ++it) {
        tc::cp_async_wait<L - 1>();  // this thread's copies of stage it have landed
        const int st = it % S;
        unsigned char *stage = dyn + st * kStageBytes;
        const unsigned char *raw = raw_base + st * (NMAT * kRawMat) + tid * 16;
#pragma unroll
        for (int i = 0; i < NMAT; ++i) {
            HalfQ2 c;
            const uint4 v = *reinterpret_cast<const uint4 *>(raw + i * kRawMat);
            c.cw = make_uint2(v.x, v.y);
            c.sc = make_uint2(v.z, v.w);
            store_half_q2(c, warp, lane, stage + i * kSub);
        }
        tc::fence_proxy_async();
        tc::mbar_arrive(&s.full[st]);
        if (it + L < nstages) ok = issue(it + L);
        tc::cp_async_commit();
        if (s.abort) break;
    }
    if (!ok) set_abort(s, p.status);
    tc::cp_async_wait_all();
}

// -------------------------------------------------------------------- gate/up
// Stage (64 of K): A_gate 16 KB, A_up 16 KB, B (256 tokens) 32 KB, plus 8 KB of
// packed codes. TMEM: D_g columns 0..255, D_u 256..511 (one accumulator pair;
// the epilogue is short).
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
    const int total = build_schedule(p, s, MT, reinterpret_cast<int *>(dyn));
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = s.tmem_base;

    if (warp < kProdWarps) {  // --------------------------------------- producers
        const MatGeom *mats[2] = {&p.gate, &p.up};
        produce<2, kGuStages, true>(p, s, dyn, total, MT, KS, mats);
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
// Stage (64 of K): A 16 KB + B (256 hidden rows) 32 KB, plus 4 KB of packed
// codes. TMEM: two 256-column accumulators (the epilogue of one tile overlaps
// the MMAs of the next).
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
    const int total = build_schedule(p, s, MT, reinterpret_cast<int *>(dyn));
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = s.tmem_base;

    if (warp < kProdWarps) {  // --------------------------------------- producers
        const MatGeom *mats[1] = {&p.down};
        produce<1, kDnStages, false>(p, s, dyn, total, MT, KS, mats);
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

// fp16 copy of the activations for the tensor cores (bf16 -> fp16 is exact for
// normal values); |x| beyond 65504 sets MOE_DEV_NONFINITE.
__global__ void __launch_bounds__(256) to_f16_kernel(const uint16_t *__restrict__ x, __half *__restrict__ y, int64_t n8,
                                                      int32_t *status) {
    bool bad = false;
    for (int64_t i = int64_t(blockIdx.x) * 256 + threadIdx.x; i < n8; i += int64_t(gridDim.x) * 256) {
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(x) + i);
        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
        uint32_t o[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float lo = bf16_lo(u[q]), hi = bf16_hi(u[q]);
            bad |= !(fabsf(lo) <= 65504.f) || !(fabsf(hi) <= 65504.f);
            const __half2 hh = __floats2half2_rn(lo, hi);
            o[q] = *reinterpret_cast<const uint32_t *>(&hh);
        }
        reinterpret_cast<uint4 *>(y)[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    if (bad) flag(status, MOE_DEV_NONFINITE);
}

std::mutex g_tc_mu;
bool g_tc_ready[64] = {};
int g_tc_sms[64] = {};

constexpr size_t kGuSmem = size_t(kGuStages) * (kGuStageBytes + 2 * kRawMat) + 1024;
constexpr size_t kDnSmem = size_t(kDnStages) * (kDnStageBytes + kRawMat) + 1024;

}  // namespace

// Launch the two grouped GEMMs (Q2); h is fp16 [T*k][f] inside the caller's workspace.
moe_status tc05_ffn_q2(const moe_qpool *W, const int32_t *slot_of, const uint16_t *x, int T, int d, int f, int E, int k,
                       const int32_t *offsets, const int32_t *sorted_tok, const int32_t *sorted_j, const int32_t *active,
                       const float *topk_w, float *out, void *ws, int32_t *dev_status, cudaStream_t stream) {
    if (reinterpret_cast<uintptr_t>(ws) % 256 || reinterpret_cast<uintptr_t>(x) % 16) return MOE_ERR_INVALID_ARG;
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
    p.x16 = reinterpret_cast<const __half *>(static_cast<unsigned char *>(ws) + tc05_x16_offset(T, k, f));
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
    const int64_t n8 = int64_t(T) * d / 8;
    to_f16_kernel<<<int(std::min<int64_t>((n8 + 255) / 256, int64_t(grid) * 8)), 256, 0, stream>>>(
        x, const_cast<__half *>(p.x16), n8, dev_status);
    tc_gateup_q2_kernel<<<grid, kTcThreads, kGuSmem, stream>>>(p);
    tc_down_q2_kernel<<<grid, kTcThreads, kDnSmem, stream>>>(p);
    return launch_status();
}

}  // namespace moe
