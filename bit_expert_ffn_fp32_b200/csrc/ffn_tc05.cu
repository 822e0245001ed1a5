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
//   producers (8 warps)  dequantise each K stage's packed codes (staged in
//                        shared memory by the TMA thread) into the fp16 A tile
//                        in tensor memory (Q2 w = s*q + m, Q3 w = s*(q-4), one
//                        fp16 rounding each); the B rows (fp16 activation rows
//                        in sorted order, or hidden rows) come straight from TMA;
//   MMA (1 thread)       issues tcgen05.mma per 16-wide K step into a TMEM
//                        accumulator;
//   TMA (2 threads)      issue the tensor-memory-accelerator loads of the
//                        packed codes and of the B rows, a few stages ahead;
//   epilogue (8 warps)   drains TMEM: h = silu(g) * u (gate/up kernel), or
//                        y_e / gate-weighted atomics (down kernel).
// Stages hand over through mbarriers; every wait is bounded and sets
// MOE_DEV_TIMEOUT instead of hanging.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>
#include <math.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "layout.h"
#include "mma_q.cuh"
#include "tc05.cuh"

namespace moe {
namespace {

constexpr int kProdWarps = 8;
constexpr int kProd = 32 * kProdWarps;  // producer threads (warps 0-7)
constexpr int kEpiWarps = 8;           // epilogue warps 8-15: TMEM lane quadrant warp % 4,
constexpr int kEpi = 32 * kEpiWarps;    //   column half (warp - 8) / 4
constexpr int kEpiWarp0 = kProdWarps;
constexpr int kMmaWarp = kProdWarps + kEpiWarps;       // 16
constexpr int kTmaWarp = kMmaWarp + 1;                 // 17: TMA loads of the packed codes
constexpr int kTmaBWarp = kMmaWarp + 2;                // 18: TMA loads of the B rows, L2 prefetch
constexpr int kTcThreads = kProd + kEpi + 96;
// Tokens per tile (MMA N, padded to 16), bounded by tensor memory: gate/up
// keeps D_gate and D_up (2 x 192 columns) plus two 64-column A stages, down
// two 192-column accumulators plus two 32-column A stages (of 512 columns).
constexpr int kTileGu = 192;
constexpr int kTileDn = 192;
constexpr int kSubB = 24576;  // B stage: 192 rows x 64 cols fp16, SW128
constexpr unsigned long long kTcWaitNs = 200ull * 1000 * 1000;
constexpr int kMaxActive = kTcMaxE;  // experts per call on this path

// Optional wait accounting (build with -DMOE_TC_TRACE): the first thread of
// each role (producer warp 0, epilogue warp 8, the MMA thread, the TMA
// thread) sums the clock64 cycles it spends in each kind of wait and writes
// the sums per CTA.
// Slots per role: 0 total, 1..5 waits (see the call sites), 6 stages/tiles.
#ifdef MOE_TC_TRACE
constexpr int kTraceCtas = 256;
__device__ unsigned long long g_tc_trace[2][kTraceCtas][4][8];
struct TcClock {
    long long v[8];
    long long t_start;
    __device__ void start() {
        for (int i = 0; i < 8; ++i) v[i] = 0;
        t_start = clock64();
    }
    __device__ long long now() const { return clock64(); }
    __device__ void add(int i, long long t0) { v[i] += clock64() - t0; }
    __device__ void count(int i) { v[i] += 1; }
    __device__ void store(int kernel, int role, bool writer) {
        v[0] = clock64() - t_start;
        if (writer && blockIdx.x < kTraceCtas)
            for (int i = 0; i < 8; ++i) g_tc_trace[kernel][blockIdx.x][role][i] = (unsigned long long)v[i];
    }
};
#else
struct TcClock {
    __device__ void start() {}
    __device__ long long now() const { return 0; }
    __device__ void add(int, long long) {}
    __device__ void count(int) {}
    __device__ void store(int, int, bool) {}
};
#endif

struct TcParams {
    const uint8_t *pool;
    int64_t slot_bytes;
    int num_slots;
    const int32_t *slot_of;
    const __half *xperm;  // [T*k][d] fp16 activation rows in sorted pair order
    int T, d, f, E, k;
    const int32_t *offsets, *sorted_tok, *sorted_j, *active;
    const float *topk_w;
    float *out;
    __half *h;  // [T*k][f] fp16 hidden rows (sorted pair order)
    int32_t *status;
    MatGeom gate, up, down;
};

constexpr int kMaxSB = 7;    // B stage slots (max over the two kernels)
constexpr int kMaxSRP = 4;   // packed-code slots
constexpr int kKeys = 512;   // schedule sort keys

// Tile order: experts from the largest to the smallest (number of 256-token
// tiles, then the size of the last tile), each expert's tiles together (N-tile
// outer, M-tile inner). Long experts start first, short ones fill the end, and
// the tiles that read the same weights run at the same time, so the weights
// come from DRAM once.
struct TcSmem {
    uint64_t fullA[2], emptyA[2], fullB[kMaxSB], emptyB[kMaxSB], fullR[kMaxSRP], emptyR[kMaxSRP], tfull[2], tempty[2];
    uint32_t tmem_base;
    int abort;
    int nexp;                          // experts with at least one tile
    int tiles_prefix[kMaxActive + 1];  // tiles before sorted expert i
    int ebeg[kMaxActive];              // sorted expert i: first sorted pair,
    int erows[kMaxActive];             //   its pair count,
    int eslot[kMaxActive];             //   its pool slot
};

// Tokens routed to active expert a that this call computes (0 if not resident).
__device__ __forceinline__ int expert_rows(const TcParams &p, int e) {
    const bool ok = e >= 0 && e < p.E;
    const int sl = ok ? p.slot_of[e] : -1;
    return (ok && sl >= 0 && sl < p.num_slots) ? p.offsets[e + 1] - p.offsets[e] : 0;
}

// Sort key (larger first): tiles (capped at 32), then the 16-token size class
// of the last tile; -1 for an expert without tokens.
__device__ __forceinline__ int sched_key(int n, int TN) {
    if (n <= 0) return -1;
    const int nt = (n + TN - 1) / TN;
    const int last = n - TN * (nt - 1);
    return (min(nt, 32) - 1) * 16 + ((last + 15) >> 4) - 1;
}

// Whole CTA: build the tile order; returns the tile count. scratch is the
// (not yet used) stage memory: kKeys + 2 * kMaxActive ints.
__device__ int build_schedule(const TcParams &p, TcSmem &s, int MT, int TN, int *scratch) {
    const int na = min(p.active[0], kMaxActive);
    const int tid = threadIdx.x, nthr = blockDim.x, lane = tid & 31;
    int *hist = scratch;                       // per key: count, then first position
    int *akey = scratch + kKeys;               // per active expert: key
    int *ord = scratch + kKeys + kMaxActive;   // sorted position -> expert id
    for (int i = tid; i < kKeys; i += nthr) hist[i] = 0;
    __syncthreads();
    for (int a = tid; a < na; a += nthr) {
        const int key = sched_key(expert_rows(p, p.active[1 + a]), TN);
        akey[a] = key;
        if (key >= 0) atomicAdd(&hist[key], 1);
    }
    __syncthreads();
    if (tid < 32) {  // descending exclusive scan over keys: lane owns keys 16*lane .. 16*lane+15
        int blk = 0;
        for (int i = 0; i < 16; ++i) blk += hist[16 * lane + i];
        int above = 0;  // experts whose key lies in a higher lane's block
        for (int l = 31; l >= 1; --l) {
            const int v = __shfl_sync(0xffffffffu, blk, l);
            if (l > lane) above += v;
        }
        int run = above;
        for (int i = 15; i >= 0; --i) {
            const int c = hist[16 * lane + i];
            hist[16 * lane + i] = run;
            run += c;
        }
        if (lane == 0) s.nexp = run;
        __syncwarp();
        // stable placement in active-index order
        for (int g0 = 0; g0 < na; g0 += 32) {
            const int a = g0 + lane;
            const int key = a < na ? akey[a] : -1;
            const unsigned peers = __match_any_sync(0xffffffffu, key);
            const int rank = __popc(peers & ((1u << lane) - 1));
            if (key >= 0) ord[hist[key] + rank] = p.active[1 + a];
            __syncwarp();
            if (key >= 0 && rank == 0) hist[key] += __popc(peers);
            __syncwarp();
        }
    }
    __syncthreads();
    const int nexp = s.nexp;
    for (int i = tid; i < nexp; i += nthr) {  // per sorted expert: rows, first pair, slot
        const int e = ord[i];
        s.erows[i] = expert_rows(p, e);
        s.ebeg[i] = p.offsets[e];
        s.eslot[i] = p.slot_of[e];
    }
    __syncthreads();
    if (tid < 32) {  // tile prefix over the sorted experts: lane owns a contiguous run
        const int per = (nexp + 31) / 32;
        const int i0 = min(nexp, lane * per), i1 = min(nexp, i0 + per);
        int sum = 0;
        for (int i = i0; i < i1; ++i) sum += MT * ((s.erows[i] + TN - 1) / TN);
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        int acc = incl - sum;
        for (int i = i0; i < i1; ++i) {
            s.tiles_prefix[i] = acc;
            acc += MT * ((s.erows[i] + TN - 1) / TN);
        }
        if (lane == 31) s.tiles_prefix[nexp] = incl;
    }
    __syncthreads();
    return s.tiles_prefix[s.nexp];
}

struct TileInfo {
    int slot, beg, rows, mi;
};

__device__ __forceinline__ TileInfo tile_info(const TcParams &p, const TcSmem &s, int tau, int MT, int TN) {
    int lo = 0, hi = s.nexp;  // last i with tiles_prefix[i] <= tau
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s.tiles_prefix[mid] <= tau) lo = mid; else hi = mid;
    }
    const int local = tau - s.tiles_prefix[lo];
    const int ni = local / MT;
    TileInfo t;
    t.slot = s.eslot[lo];
    t.mi = local - ni * MT;
    t.beg = s.ebeg[lo] + TN * ni;
    t.rows = min(TN, s.erows[lo] - TN * ni);
    return t;
}

// The packed codes (8 B) and scale entry (8 B) of one block of one lane chunk:
// block bb of the pair, rows g and g+8, {s(g), s(g+8), m(g), m(g+8)}.
struct HalfQ2 {
    uint2 cw, sc;
};

// Dequantise one block of a lane chunk (rows g and g+8, k = 16i + 8s + 2t + h
// for register slot rho = 2i + s) into fp16 pairs: v[2*rho] row g, v[2*rho+1]
// row g+8; w = s*q + m (q made exact in fp16 by the 1024-offset trick, then
// one fused multiply-add).
__device__ __forceinline__ void dequant_half_q2(const HalfQ2 &c, uint32_t (&v)[16]) {
    const __half2 k1024 = __half2half2(__ushort_as_half(0x6400));
    const __half2 s01 = *reinterpret_cast<const __half2 *>(&c.sc.x);
    const __half2 m01 = *reinterpret_cast<const __half2 *>(&c.sc.y);
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const uint32_t w = r ? c.cw.y : c.cw.x;
        const __half2 s2 = r ? __high2half2(s01) : __low2half2(s01);
        const __half2 m2 = r ? __high2half2(m01) : __low2half2(m01);
#pragma unroll
        for (int rho = 0; rho < 8; ++rho) {
            const uint32_t qbits = ((w >> (2 * rho)) & 0x00030003u) | 0x64006400u;
            const __half2 q = __hsub2(*reinterpret_cast<const __half2 *>(&qbits), k1024);
            const __half2 wv = __hfma2(s2, q, m2);
            v[2 * rho + r] = *reinterpret_cast<const uint32_t *>(&wv);
        }
    }
}

// Dequantise block BQ of a Q3 lane chunk (the 12 words of a block quad; s01 =
// {s(g), s(g+8)} of the block) into fp16 pairs in the same register order as
// dequant_half_q2: w = s*(q-4), q-4 exact in fp16 (1024-offset trick), one
// rounding in the product.
template <int BQ>
__device__ __forceinline__ void dequant_block_q3(const uint32_t (&W)[12], uint32_t s01, uint32_t (&v)[16]) {
    const __half2 k1028 = __half2half2(__ushort_as_half(0x6404));
    const __half2 s2x = *reinterpret_cast<const __half2 *>(&s01);
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const __half2 s2 = r ? __high2half2(s2x) : __low2half2(s2x);
#pragma unroll
        for (int rho = 0; rho < 8; ++rho) {
            const int u = 8 * BQ + rho;
            const uint32_t qbits = (q3_reg(W, u, r) >> q3_exp(u)) | 0x64006400u;
            const __half2 q = __hsub2(*reinterpret_cast<const __half2 *>(&qbits), k1028);
            const __half2 wv = __hmul2(s2, q);
            v[2 * rho + r] = *reinterpret_cast<const uint32_t *>(&wv);
        }
    }
}

// Block bq (run time) of the quad; every register index stays a compile-time constant.
__device__ __forceinline__ void dequant_q3(const uint32_t (&W)[12], const uint32_t (&s)[4], int bq,
                                           uint32_t (&v)[16]) {
    switch (bq) {
        case 0: dequant_block_q3<0>(W, s[0], v); break;
        case 1: dequant_block_q3<1>(W, s[1], v); break;
        case 2: dequant_block_q3<2>(W, s[2], v); break;
        default: dequant_block_q3<3>(W, s[3], v); break;
    }
}

__device__ __forceinline__ void set_abort(TcSmem &s, int32_t *status) {
    if (atomicExch(&s.abort, 1) == 0) flag(status, MOE_DEV_TIMEOUT);
}

// Packed bytes of one code unit of a 128-row tile, per matrix: a block pair
// (two K stages) for Q2, 8 row groups x 32 lanes x 16 B of codes, then 8 row
// groups x 8 x 16 B of scales; a block quad (four K stages) for Q3, 8 row
// groups x 3 x 32 lanes x 16 B of codes, then 8 row groups x 2 x 8 x 8 B of
// scales.
template <int FMT>
struct RawUnit {
    static constexpr int kStages = FMT == 2 ? 2 : 4;
    static constexpr int kCodes = FMT == 2 ? 8 * 512 : 8 * 1536;
    static constexpr int kMat = kCodes + 8 * 128;
};

// Shared-memory rings of a kernel: SB B stages (192 rows x 64 fp16) and SRP
// slots of packed A bytes (one code unit each). The dequantised A stages live
// in tensor memory.
template <int FMT, int NMAT, int SB, int SRP>
struct Rings {
    static constexpr int kRaw = NMAT * RawUnit<FMT>::kMat;
    static constexpr int kBytes = SB * kSubB + SRP * kRaw;
    __device__ static unsigned char *b(unsigned char *dyn, int it) { return dyn + (it % SB) * kSubB; }
    __device__ static unsigned char *raw(unsigned char *dyn, int pp) { return dyn + SB * kSubB + (pp % SRP) * kRaw; }
};

// Tensor maps of the packed weights, per matrix. Q2: codes as uint32 [slot][row
// group][pair * 128 words], scales as [slot][row group][pair * 32 words]. Q3:
// codes as uint32 [slot][row group][quad * 3 sub-chunks][128 words], scales as
// [slot][row group][quad * 32 words].
struct RawMaps {
    CUtensorMap code[2], scale[2];
};

// Walks this CTA's (tile, step) sequence; tau advances by the grid size.
struct StageCursor {
    int tau, ks;
};

// TMA threads (lane 0 of warps 17 and 18), each walking this CTA's stages in
// order and blocking only on the slot it refills next:
//   A codes  (warp 17) one load of codes and one of scales per matrix and
//            code unit (two stages Q2, four Q3) into slot pp % SRP once every
//            producer is done with it (emptyR); complete on fullR;
//   B rows   (warp 18) TMA loads of the tile's rows, 64 per box, into B slot
//            it % SB once the MMA has released it (emptyB); complete on
//            fullB. On entering a tile it asks the L2 for the next tile.
template <int FMT, int NMAT, int SA, int SB, int SRP>
__device__ __forceinline__ void issue_codes(const TcParams &p, TcSmem &s, unsigned char *dyn, int total, int MT, int TN,
                                            int KS, const RawMaps &rm) {
    using R = Rings<FMT, NMAT, SB, SRP>;
    using U = RawUnit<FMT>;
    const int PS = KS / U::kStages;
    const int mine = blockIdx.x < total ? (total - int(blockIdx.x) + int(gridDim.x) - 1) / int(gridDim.x) : 0;
    const int npairs = mine * PS;
    TcClock ck;
    ck.start();
#pragma unroll
    for (int i = 0; i < NMAT; ++i) {
        tc::prefetch_tensormap(&rm.code[i]);
        tc::prefetch_tensormap(&rm.scale[i]);
    }
    int tau = blockIdx.x, pk = 0;
    TileInfo t{};
    if (mine > 0) t = tile_info(p, s, tau, MT, TN);
    bool ok = true;
#pragma unroll 1
    for (int pr = 0; pr < npairs && !s.abort; ++pr) {
        const long long t0 = ck.now();
        if (!tc::mbar_wait(&s.emptyR[pr % SRP], ((pr / SRP) & 1) ^ 1, kTcWaitNs)) {
            ok = false;
            break;
        }
        ck.add(1, t0);
        const long long t1 = ck.now();
        unsigned char *raw = R::raw(dyn, pr);
        uint64_t *bar = &s.fullR[pr % SRP];
        tc::mbar_arrive_expect_tx(bar, uint32_t(NMAT * U::kMat));
#pragma unroll
        for (int i = 0; i < NMAT; ++i) {
            if (FMT == 2)
                tc::tma_load_3d(raw + i * U::kMat, &rm.code[i], 128 * pk, 8 * t.mi, t.slot, bar);
            else
                tc::tma_load_4d(raw + i * U::kMat, &rm.code[i], 0, 3 * pk, 8 * t.mi, t.slot, bar);
            tc::tma_load_3d(raw + i * U::kMat + U::kCodes, &rm.scale[i], 32 * pk, 8 * t.mi, t.slot, bar);
        }
        ck.add(3, t1);
        ck.count(6);
        if (++pk == PS) {
            pk = 0;
            tau += gridDim.x;
            if (tau < total) t = tile_info(p, s, tau, MT, TN);
        }
    }
    if (!ok) set_abort(s, p.status);
    ck.store(NMAT == 2 ? 0 : 1, 3, true);
}

template <int FMT, int NMAT, int SA, int SB, int SRP>
__device__ __forceinline__ void issue_rows(const TcParams &p, TcSmem &s, unsigned char *dyn, int total, int MT, int TN,
                                           int KS, const void *tmap_b, const __half *bsrc) {
    using R = Rings<FMT, NMAT, SB, SRP>;
    const int mine = blockIdx.x < total ? (total - int(blockIdx.x) + int(gridDim.x) - 1) / int(gridDim.x) : 0;
    const int nstages = mine * KS;
    tc::prefetch_tensormap(tmap_b);
    int tau = blockIdx.x, ks = 0;
    TileInfo t{};
    if (mine > 0) t = tile_info(p, s, tau, MT, TN);
    bool ok = true;
#pragma unroll 1
    for (int pb = 0; pb < nstages && !s.abort; ++pb) {
        if (!tc::mbar_wait(&s.emptyB[pb % SB], ((pb / SB) & 1) ^ 1, kTcWaitNs)) {
            ok = false;
            break;
        }
        unsigned char *bsub = R::b(dyn, pb);
        uint64_t *bar = &s.fullB[pb % SB];
        const int nbox = (t.rows + 63) >> 6;
        tc::mbar_arrive_expect_tx(bar, uint32_t(nbox) * 8192u);
        for (int j = 0; j < nbox; ++j) tc::tma_load_2d(bsub + j * 8192, tmap_b, 64 * ks, t.beg + 64 * j, bar);
        if (++ks == KS) {
            ks = 0;
            tau += gridDim.x;
            if (tau < total) t = tile_info(p, s, tau, MT, TN);
        }
    }
    if (!ok) set_abort(s, p.status);
}

// Producer warps (0-7): warp w owns row group rgl = 2(w%4) + w/4 of the
// 128-row tile (its tensor-memory lane quadrant is w%4). For each stage, once
// the code unit's packed bytes have landed (fullR), each thread loads its lane
// chunk (rows g, g+8 of the row group; k-slots of t) -- Q2 one block's 8 B of
// codes and scales per stage, releasing the slot (emptyR) after the pair's
// second block; Q3 the quad's 48 B of codes and 16 B of scales at its first
// block, releasing the slot at once -- and dequantises into registers; once
// the MMA has released the A stage (emptyA) it stores the chunk to the stage's
// TMEM columns (lane g / g+8, column 4*rho + t = k/2) and arrives on fullA. a_col0: TMEM column of A
// stage 0, matrix 0; stages are 32*NMAT columns apart.
template <int FMT, int NMAT, int SA, int SB, int SRP>
__device__ __forceinline__ void produce(const TcParams &p, TcSmem &s, unsigned char *dyn, int total, int KS,
                                        uint32_t tmem, int a_col0) {
    using R = Rings<FMT, NMAT, SB, SRP>;
    using U = RawUnit<FMT>;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int rgl = 2 * (warp & 3) + (warp >> 2);
    const uint32_t ta = tmem + (uint32_t(16 * rgl) << 16) + uint32_t(a_col0);
    const int mine = blockIdx.x < total ? (total - int(blockIdx.x) + int(gridDim.x) - 1) / int(gridDim.x) : 0;
    const int nstages = mine * KS;
    TcClock ck;
    ck.start();
    bool ok = true;
    uint32_t w3[NMAT][12], s3[NMAT][4];  // Q3: the quad's lane chunk, kept for its four stages
#pragma unroll 1
    for (int it = 0; it < nstages; ++it) {
        const int pp = it / U::kStages, bb = it % U::kStages;
        long long t0 = ck.now();
        if (bb == 0 && !tc::mbar_wait(&s.fullR[pp % SRP], (pp / SRP) & 1, kTcWaitNs)) {
            ok = false;
            break;
        }
        ck.add(1, t0);
        t0 = ck.now();
        const unsigned char *raw = R::raw(dyn, pp);
        uint32_t v[NMAT][16];
        if (FMT == 2) {
            HalfQ2 c[NMAT];  // both matrices' bytes first, then both dequantised together
#pragma unroll
            for (int i = 0; i < NMAT; ++i) {
                c[i].cw = *reinterpret_cast<const uint2 *>(raw + i * U::kMat + rgl * 512 + lane * 16 + 8 * bb);
                c[i].sc = *reinterpret_cast<const uint2 *>(raw + i * U::kMat + U::kCodes + rgl * 128 +
                                                           (lane >> 2) * 16 + 8 * bb);
            }
            if (bb) tc::mbar_arrive(&s.emptyR[pp % SRP]);  // both blocks of the pair are in registers
            // dequantise into registers while the MMA may still be reading this A stage
#pragma unroll
            for (int i = 0; i < NMAT; ++i) dequant_half_q2(c[i], v[i]);
        } else {
            if (bb == 0) {
#pragma unroll
                for (int i = 0; i < NMAT; ++i) {
                    const unsigned char *cb = raw + i * U::kMat + rgl * 1536 + lane * 16;
#pragma unroll
                    for (int sub = 0; sub < 3; ++sub) {
                        const uint4 q = *reinterpret_cast<const uint4 *>(cb + sub * 512);
                        w3[i][4 * sub + 0] = q.x;
                        w3[i][4 * sub + 1] = q.y;
                        w3[i][4 * sub + 2] = q.z;
                        w3[i][4 * sub + 3] = q.w;
                    }
                    // scale entries of the quad's two pairs: {s(g), s(g+8)} per block
                    const unsigned char *sb = raw + i * U::kMat + U::kCodes + rgl * 128 + (lane >> 2) * 8;
                    const uint2 a = *reinterpret_cast<const uint2 *>(sb);
                    const uint2 b = *reinterpret_cast<const uint2 *>(sb + 64);
                    s3[i][0] = a.x;
                    s3[i][1] = a.y;
                    s3[i][2] = b.x;
                    s3[i][3] = b.y;
                }
                tc::mbar_arrive(&s.emptyR[pp % SRP]);  // the whole quad is in registers
            }
#pragma unroll
            for (int i = 0; i < NMAT; ++i) dequant_q3(w3[i], s3[i], bb, v[i]);
        }
        ck.add(4, t0);
        t0 = ck.now();
        if (!tc::mbar_wait(&s.emptyA[it % SA], ((it / SA) & 1) ^ 1, kTcWaitNs)) {
            ok = false;
            break;
        }
        tc::fence_after();
        ck.add(2, t0);
        t0 = ck.now();
        const long long t2 = ck.now();
#pragma unroll
        for (int i = 0; i < NMAT; ++i) tc::tmem_st16x128_x8(ta + uint32_t((it % SA) * 32 * NMAT + 32 * i), v[i]);
        ck.add(3, t2);
        const long long t3 = ck.now();
        tc::tmem_st_wait();
        ck.add(5, t3);
        tc::fence_before();
        tc::mbar_arrive(&s.fullA[it % SA]);
        ck.add(4, t0);
        ck.count(6);
        if (s.abort) break;
    }
    if (!ok) set_abort(s, p.status);
    ck.store(NMAT == 2 ? 0 : 1, 0, tid == 0);
}

// Barrier set-up shared by both kernels (thread 0), then TMEM allocation
// (MMA warp) and the schedule (whole CTA).
template <int SA, int SB, int SRP>
__device__ __forceinline__ void init_barriers(TcSmem &s, int acc_bufs) {
    for (int i = 0; i < SRP; ++i) {
        tc::mbar_init(&s.fullR[i], 1);
        tc::mbar_init(&s.emptyR[i], kProd);
    }
    for (int i = 0; i < SA; ++i) {
        tc::mbar_init(&s.fullA[i], kProd);
        tc::mbar_init(&s.emptyA[i], 1);
    }
    for (int i = 0; i < SB; ++i) {
        tc::mbar_init(&s.fullB[i], 1);
        tc::mbar_init(&s.emptyB[i], 1);
    }
    for (int i = 0; i < acc_bufs; ++i) {
        tc::mbar_init(&s.tfull[i], 1);
        tc::mbar_init(&s.tempty[i], kEpi);
    }
    s.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// MMA thread: wait for stage it's A and B, then hand both slots back when the
// MMAs that read them have completed.
template <int SA, int SB>
__device__ __forceinline__ bool mma_wait_stage(TcSmem &s, int it, TcClock &ck) {
    long long t0 = ck.now();
    if (!tc::mbar_wait(&s.fullA[it % SA], (it / SA) & 1, kTcWaitNs)) return false;
    ck.add(1, t0);
    t0 = ck.now();
    if (!tc::mbar_wait(&s.fullB[it % SB], (it / SB) & 1, kTcWaitNs)) return false;
    ck.add(2, t0);
    ck.count(6);
    tc::fence_after();
    return true;
}
template <int SA, int SB>
__device__ __forceinline__ void mma_release_stage(TcSmem &s, int it) {
    tc::mma_commit(&s.emptyA[it % SA]);
    tc::mma_commit(&s.emptyB[it % SB]);
}

// -------------------------------------------------------------------- gate/up
// Shared memory: 5 B stages (up to 192 tokens, 24 KB each), packed-code slots
// (Q2: 4 of one block pair, 10 KB each; Q3: 2 of one block quad, 26 KB each),
// 1 KB of h staging per epilogue warp. TMEM: D_gate columns 0..191, D_up
// 192..383 (one accumulator pair), A stages at 384 and 448 (gate 32 columns,
// then up 32 columns).
constexpr int kGuSA = 2, kGuSB = 5;
template <int FMT>
struct GuSR {
    static constexpr int v = FMT == 2 ? 4 : 2;
};
constexpr int kHStage = 1024;  // per epilogue warp: 16 tokens x 32 rows of h (fp16)
constexpr int kGuColU = kTileGu, kGuColA = 2 * kTileGu;
template <int FMT>
using GuRings = Rings<FMT, 2, kGuSB, GuSR<FMT>::v>;

template <int FMT>
__global__ void __launch_bounds__(kTcThreads, 1)
    tc_gateup_kernel(const __grid_constant__ TcParams p, const __grid_constant__ CUtensorMap tmap_b,
                     const __grid_constant__ RawMaps rm) {
    constexpr int kGuSR = GuSR<FMT>::v;
    extern __shared__ __align__(1024) unsigned char dyn_raw[];
    unsigned char *dyn =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(dyn_raw) + 1023) & ~uintptr_t(1023));
    __shared__ TcSmem s;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int MT = p.f / 128, KS = p.d / 64, TN = kTileGu;
    unsigned char *hstage = dyn + GuRings<FMT>::kBytes;  // epilogue staging of h
    if (tid == 0) init_barriers<kGuSA, kGuSB, kGuSR>(s, 1);
    if (warp == kMmaWarp) tc::tmem_alloc(&s.tmem_base, 512);
    const int total = build_schedule(p, s, MT, TN, reinterpret_cast<int *>(dyn));
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = s.tmem_base;

    if (warp < kProdWarps) {  // --------------------------------------- producers
        produce<FMT, 2, kGuSA, kGuSB, kGuSR>(p, s, dyn, total, KS, tmem, kGuColA);
    } else if (warp < kMmaWarp) {  // ---------------------------------- epilogue
        const int q = warp & 3, half = (warp - kEpiWarp0) >> 2;  // TMEM lane quadrant, column half
        int tcount = 0;
        bool too_big = false;
        TcClock ck;
        ck.start();
        for (int tau = blockIdx.x; tau < total && !s.abort; tau += gridDim.x, ++tcount) {
            const TileInfo ti = tile_info(p, s, tau, MT, TN);
            const long long t0 = ck.now();
            if (!tc::mbar_wait_sleep(&s.tfull[0], tcount & 1, kTcWaitNs, 128)) {
                set_abort(s, p.status);
                break;
            }
            ck.add(1, t0);
            ck.count(6);
            tc::fence_after();
            // rows 128mi + 32q + lane of h for 16 tokens at a time: staged in this
            // warp's 1 KB ([token][32 rows] fp16), then written as 64-byte pieces
            // (16 bytes per lane) of the tokens' h rows
            const uint32_t tg = tmem + (uint32_t(32 * q) << 16);
            __half *hs = reinterpret_cast<__half *>(hstage + (warp - kEpiWarp0) * kHStage);
            __half *hrow0 = p.h + int64_t(ti.beg) * p.f + 128 * ti.mi + 32 * q;
            for (int c0 = 16 * half; c0 < ti.rows; c0 += 32) {
                float g[16], u[16];
                const long long t1 = ck.now();
                tc::tmem_ld16(tg + c0, g);
                tc::tmem_ld16(tg + kGuColU + c0, u);
                ck.add(2, t1);
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float hv = __fdividef(g[j], 1.0f + __expf(-g[j])) * u[j];
                    too_big |= c0 + j < ti.rows && !(fabsf(hv) <= 65504.f);
                    hs[j * 32 + lane] = __float2half_rn(hv);
                }
                __syncwarp();
#pragma unroll
                for (int pass = 0; pass < 2; ++pass) {
                    const int j = 8 * pass + (lane >> 2), ch = lane & 3;
                    if (c0 + j < ti.rows)
                        *reinterpret_cast<uint4 *>(hrow0 + int64_t(c0 + j) * p.f + 8 * ch) =
                            *reinterpret_cast<const uint4 *>(hs + j * 32 + 8 * ch);
                }
                __syncwarp();
            }
            tc::fence_before();
            tc::mbar_arrive(&s.tempty[0]);
        }
        if (too_big) flag(p.status, MOE_DEV_NONFINITE);
        ck.store(0, 1, warp == kEpiWarp0 && lane == 0);
    } else if (warp == kTmaWarp) {  // -------------------------------------- TMA
        if (lane == 0) issue_codes<FMT, 2, kGuSA, kGuSB, kGuSR>(p, s, dyn, total, MT, TN, KS, rm);
    } else if (warp == kTmaBWarp) {
        if (lane == 0) issue_rows<FMT, 2, kGuSA, kGuSB, kGuSR>(p, s, dyn, total, MT, TN, KS, &tmap_b, p.xperm);
    } else if (lane == 0) {  // --------------------------------------------- MMA
        int it = 0, tcount = 0;
        bool ok = true;
        TcClock ck;
        ck.start();
        for (int tau = blockIdx.x; tau < total && ok && !s.abort; tau += gridDim.x, ++tcount) {
            const TileInfo ti = tile_info(p, s, tau, MT, TN);
            const int npad = (ti.rows + 15) & ~15;
            const uint32_t idesc = tc::idesc_f16(128, npad);
            const long long t0 = ck.now();
            if (!tc::mbar_wait(&s.tempty[0], (tcount & 1) ^ 1, kTcWaitNs)) {
                ok = false;
                break;
            }
            ck.add(3, t0);
            tc::fence_after();
            const uint32_t dg = tmem, du = tmem + kGuColU;
            for (int ks = 0; ks < KS; ++ks, ++it) {
                if (!mma_wait_stage<kGuSA, kGuSB>(s, it, ck)) {
                    ok = false;
                    break;
                }
                const uint32_t a = tmem + uint32_t(kGuColA + (it % kGuSA) * 64);  // gate, then up at +32
                const uint32_t b = tc::smem_u32(GuRings<FMT>::b(dyn, it));
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t bd = tc::desc_sw128(b + 32 * kk);
                    const uint32_t acc = (ks | kk) ? 1u : 0u;
                    tc::mma_f16_ta(dg, a + 8 * kk, bd, idesc, acc);
                    tc::mma_f16_ta(du, a + 32 + 8 * kk, bd, idesc, acc);
                }
                mma_release_stage<kGuSA, kGuSB>(s, it);
            }
            if (ok) tc::mma_commit(&s.tfull[0]);
        }
        if (!ok) set_abort(s, p.status);
        ck.store(0, 2, true);
    }
    tc::fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc::fence_after();
        tc::tmem_dealloc(tmem, 512);
    }
}

// ----------------------------------------------------------------------- down
// Shared memory: 7 B stages (up to 192 hidden rows, 24 KB each), packed-code
// slots (Q2: 4 of one block pair, 5 KB each; Q3: 2 of one block quad, 13 KB
// each). TMEM: two 192-column accumulators at 0 and 192 (the epilogue of one
// tile overlaps the MMAs of the next), A stages at 384 and 416.
constexpr int kDnSA = 2, kDnSB = 7;
template <int FMT>
struct DnSR {
    static constexpr int v = FMT == 2 ? 4 : 2;
};
constexpr int kDnColA = 2 * kTileDn;
template <int FMT>
using DnRings = Rings<FMT, 1, kDnSB, DnSR<FMT>::v>;

template <int FMT>
__global__ void __launch_bounds__(kTcThreads, 1)
    tc_down_kernel(const __grid_constant__ TcParams p, const __grid_constant__ CUtensorMap tmap_b,
                   const __grid_constant__ RawMaps rm) {
    constexpr int kDnSR = DnSR<FMT>::v;
    extern __shared__ __align__(1024) unsigned char dyn_raw[];
    unsigned char *dyn =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(dyn_raw) + 1023) & ~uintptr_t(1023));
    __shared__ TcSmem s;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int MT = p.d / 128, KS = p.f / 64, TN = kTileDn;
    if (tid == 0) init_barriers<kDnSA, kDnSB, kDnSR>(s, 2);
    if (warp == kMmaWarp) tc::tmem_alloc(&s.tmem_base, 512);
    const int total = build_schedule(p, s, MT, TN, reinterpret_cast<int *>(dyn));
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = s.tmem_base;

    if (warp < kProdWarps) {  // --------------------------------------- producers
        produce<FMT, 1, kDnSA, kDnSB, kDnSR>(p, s, dyn, total, KS, tmem, kDnColA);
    } else if (warp < kMmaWarp) {  // ---------------------------------- epilogue
        const int q = warp & 3, half = (warp - kEpiWarp0) >> 2;
        int tcount = 0;
        TcClock ck;
        ck.start();
        for (int tau = blockIdx.x; tau < total && !s.abort; tau += gridDim.x, ++tcount) {
            const TileInfo ti = tile_info(p, s, tau, MT, TN);
            const int b = tcount & 1;
            const uint32_t ph = (tcount >> 1) & 1;
            const long long t0 = ck.now();
            if (!tc::mbar_wait_sleep(&s.tfull[b], ph, kTcWaitNs, 128)) {
                set_abort(s, p.status);
                break;
            }
            ck.add(1, t0);
            ck.count(6);
            tc::fence_after();
            const int drow = 128 * ti.mi + 32 * q + lane;
            const uint32_t td = tmem + (uint32_t(32 * q) << 16) + uint32_t(b * kTileDn);
            for (int c0 = 16 * half; c0 < ti.rows; c0 += 32) {
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
        ck.store(1, 1, warp == kEpiWarp0 && lane == 0);
    } else if (warp == kTmaWarp) {  // -------------------------------------- TMA
        if (lane == 0) issue_codes<FMT, 1, kDnSA, kDnSB, kDnSR>(p, s, dyn, total, MT, TN, KS, rm);
    } else if (warp == kTmaBWarp) {
        if (lane == 0) issue_rows<FMT, 1, kDnSA, kDnSB, kDnSR>(p, s, dyn, total, MT, TN, KS, &tmap_b, p.h);
    } else if (lane == 0) {  // --------------------------------------------- MMA
        int it = 0, tcount = 0;
        bool ok = true;
        TcClock ck;
        ck.start();
        for (int tau = blockIdx.x; tau < total && ok && !s.abort; tau += gridDim.x, ++tcount) {
            const TileInfo ti = tile_info(p, s, tau, MT, TN);
            const int npad = (ti.rows + 15) & ~15;
            const uint32_t idesc = tc::idesc_f16(128, npad);
            const int b = tcount & 1;
            const uint32_t phb = (tcount >> 1) & 1;
            const long long t0 = ck.now();
            if (!tc::mbar_wait(&s.tempty[b], phb ^ 1, kTcWaitNs)) {
                ok = false;
                break;
            }
            ck.add(3, t0);
            tc::fence_after();
            const uint32_t dd = tmem + uint32_t(b * kTileDn);
            for (int ks = 0; ks < KS; ++ks, ++it) {
                if (!mma_wait_stage<kDnSA, kDnSB>(s, it, ck)) {
                    ok = false;
                    break;
                }
                const uint32_t a = tmem + uint32_t(kDnColA + (it % kDnSA) * 32);
                const uint32_t bb = tc::smem_u32(DnRings<FMT>::b(dyn, it));
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_f16_ta(dd, a + 8 * kk, tc::desc_sw128(bb + 32 * kk), idesc, (ks | kk) ? 1u : 0u);
                mma_release_stage<kDnSA, kDnSB>(s, it);
            }
            if (ok) tc::mma_commit(&s.tfull[b]);
        }
        if (!ok) set_abort(s, p.status);
        ck.store(1, 2, true);
    }
    tc::fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc::fence_after();
        tc::tmem_dealloc(tmem, 512);
    }
}

// Activation rows in sorted pair order, as fp16 for the tensor cores:
// xperm[s] = x[sorted_tok[s]] (bf16 -> fp16 is exact for normal values);
// |x| beyond 65504 sets MOE_DEV_NONFINITE. One CTA per row at a time.
__global__ void __launch_bounds__(256) gather_f16_kernel(const uint16_t *__restrict__ x,
                                                          const int32_t *__restrict__ sorted_tok, int d, int64_t rows,
                                                          __half *__restrict__ y, int32_t *status) {
    bool bad = false;
    const int n8 = d / 8;
    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
        const int64_t t = sorted_tok[r];
        const uint4 *src = reinterpret_cast<const uint4 *>(x + t * d);
        uint4 *dst = reinterpret_cast<uint4 *>(y + r * d);
        for (int c = threadIdx.x; c < n8; c += blockDim.x) {
            const uint4 v = __ldg(src + c);
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
            uint32_t o[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float lo = bf16_lo(u[q]), hi = bf16_hi(u[q]);
                bad |= !(fabsf(lo) <= 65504.f) || !(fabsf(hi) <= 65504.f);
                const __half2 hh = __floats2half2_rn(lo, hi);
                o[q] = *reinterpret_cast<const uint32_t *>(&hh);
            }
            dst[c] = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
    if (bad) flag(status, MOE_DEV_NONFINITE);
}

std::mutex g_tc_mu;
bool g_tc_ready[64] = {};
int g_tc_sms[64] = {};
PFN_cuTensorMapEncodeTiled_v12000 g_encode_tiled = nullptr;

// 2D fp16 tensor [rows][inner] (row pitch inner * 2 bytes) read in boxes of
// box_rows x 64 with the 128-byte swizzle the MMA descriptors expect.
bool f16_map(CUtensorMap *m, const void *base, int64_t inner, int64_t rows, uint32_t box_rows) {
    const cuuint64_t dims[2] = {cuuint64_t(inner), cuuint64_t(rows)};
    const cuuint64_t strides[1] = {cuuint64_t(inner) * 2};
    const cuuint32_t box[2] = {64, box_rows};
    const cuuint32_t es[2] = {1, 1};
    return g_encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(base), dims, strides, box, es,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3D uint32 view [slots][row groups][words] of one region (codes or scales) of
// matrix m in every pool slot, read in boxes of 8 row groups x box_words.
bool raw_map(CUtensorMap *map, const uint8_t *pool, int64_t slot_bytes, int num_slots, uint64_t region_off,
             int64_t words_per_group, int groups, uint32_t box_words) {
    const cuuint64_t dims[3] = {cuuint64_t(words_per_group), cuuint64_t(groups), cuuint64_t(num_slots)};
    const cuuint64_t strides[2] = {cuuint64_t(words_per_group) * 4, cuuint64_t(slot_bytes)};
    const cuuint32_t box[3] = {box_words, 8, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    return g_encode_tiled(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<uint8_t *>(pool + region_off), dims,
                          strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Q3 codes as a 4D uint32 view [slots][row groups][quads * 3 sub-chunks][128
// words], read in boxes of one quad's 3 sub-chunks x 8 row groups (12 KB).
bool q3_code_map(CUtensorMap *map, const uint8_t *pool, int64_t slot_bytes, int num_slots, const MatGeom &m) {
    const cuuint64_t dims[4] = {128, cuuint64_t(m.NB / 4) * 3, cuuint64_t(m.NG), cuuint64_t(num_slots)};
    const cuuint64_t strides[3] = {512, cuuint64_t(m.NB / 4) * 1536, cuuint64_t(slot_bytes)};
    const cuuint32_t box[4] = {128, 3, 8, 1};
    const cuuint32_t es[4] = {1, 1, 1, 1};
    return g_encode_tiled(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, const_cast<uint8_t *>(pool + m.codes_off), dims,
                          strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int FMT>
bool raw_maps(RawMaps *rm, const TcParams &p, const MatGeom *const *mats, int nmat) {
    for (int i = 0; i < nmat; ++i) {
        const MatGeom &m = *mats[i];
        const bool codes = FMT == 2 ? raw_map(&rm->code[i], p.pool, p.slot_bytes, p.num_slots, m.codes_off,
                                              int64_t(m.NB / 2) * 128, m.NG, 128)
                                    : q3_code_map(&rm->code[i], p.pool, p.slot_bytes, p.num_slots, m);
        // scales: 32 words per code unit (Q2 one pair of 16 B entries, Q3 two pairs of 8 B entries)
        if (!codes || !raw_map(&rm->scale[i], p.pool, p.slot_bytes, p.num_slots, m.scales_off,
                               int64_t(m.NB / 2) * (FMT == 2 ? 32 : 16), m.NG, 32))
            return false;
    }
    return true;
}

template <int FMT>
constexpr size_t gu_smem() { return size_t(GuRings<FMT>::kBytes) + size_t(kEpiWarps) * kHStage + 1024; }
template <int FMT>
constexpr size_t dn_smem() { return size_t(DnRings<FMT>::kBytes) + 1024; }
static_assert(kDnSB <= kMaxSB && kGuSB <= kMaxSB && DnSR<2>::v <= kMaxSRP && GuSR<2>::v <= kMaxSRP &&
                  DnSR<3>::v <= kMaxSRP && GuSR<3>::v <= kMaxSRP,
              "ring larger than its barrier array");
static_assert(size_t(kKeys + 2 * kMaxActive) * 4 <= size_t(GuRings<2>::kBytes) &&
                  size_t(kKeys + 2 * kMaxActive) * 4 <= size_t(DnRings<2>::kBytes) &&
                  size_t(kKeys + 2 * kMaxActive) * 4 <= size_t(GuRings<3>::kBytes) &&
                  size_t(kKeys + 2 * kMaxActive) * 4 <= size_t(DnRings<3>::kBytes),
              "schedule scratch does not fit the stage memory");
static_assert(gu_smem<2>() + sizeof(TcSmem) <= 232448 && dn_smem<2>() + sizeof(TcSmem) <= 232448 &&
                  gu_smem<3>() + sizeof(TcSmem) <= 232448 && dn_smem<3>() + sizeof(TcSmem) <= 232448,
              "shared memory above the 227 KB a CTA may use");

template <int FMT>
bool set_smem_attrs() {
    return cudaFuncSetAttribute(tc_gateup_kernel<FMT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                int(gu_smem<FMT>())) == cudaSuccess &&
           cudaFuncSetAttribute(tc_down_kernel<FMT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                int(dn_smem<FMT>())) == cudaSuccess;
}

template <int FMT>
moe_status tc05_ffn_fmt(const moe_qpool *W, const int32_t *slot_of, const uint16_t *x, int T, int d, int f, int E,
                        int k, const int32_t *offsets, const int32_t *sorted_tok, const int32_t *sorted_j,
                        const int32_t *active, const float *topk_w, float *out, void *ws, int32_t *dev_status,
                        cudaStream_t stream) {
    if (reinterpret_cast<uintptr_t>(ws) % 256 || reinterpret_cast<uintptr_t>(x) % 16) return MOE_ERR_INVALID_ARG;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    {
        std::lock_guard<std::mutex> lock(g_tc_mu);
        if (!g_tc_ready[dev]) {
            if (!set_smem_attrs<2>() || !set_smem_attrs<3>() ||
                cudaDeviceGetAttribute(&g_tc_sms[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
                cudaGetLastError();
                return MOE_ERR_CUDA;
            }
            if (!g_encode_tiled) {
                void *fn = nullptr;
                cudaDriverEntryPointQueryResult q;
                if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) !=
                        cudaSuccess ||
                    q != cudaDriverEntryPointSuccess || !fn) {
                    cudaGetLastError();
                    return MOE_ERR_CUDA;
                }
                g_encode_tiled = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
            }
            g_tc_ready[dev] = true;
        }
    }
    const ExpertGeom eg = expert_geom(FMT, d, f);
    TcParams p;
    p.pool = static_cast<const uint8_t *>(W->base);
    p.slot_bytes = W->slot_bytes;
    p.num_slots = W->num_slots;
    p.slot_of = slot_of;
    p.xperm = reinterpret_cast<const __half *>(static_cast<unsigned char *>(ws) + tc05_xperm_offset(T, k, f));
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
    const int64_t pairs = int64_t(T) * k;
    gather_f16_kernel<<<int(std::min<int64_t>(pairs, int64_t(grid) * 8)), 256, 0, stream>>>(
        x, sorted_tok, d, pairs, const_cast<__half *>(p.xperm), dev_status);
    CUtensorMap map_x, map_h;  // B operands: activation rows (gate/up), hidden rows (down)
    RawMaps rm_gu, rm_dn;
    const MatGeom *gu[2] = {&p.gate, &p.up}, *dn[1] = {&p.down};
    if (!f16_map(&map_x, p.xperm, d, pairs, 64) || !f16_map(&map_h, p.h, f, pairs, 64) ||
        !raw_maps<FMT>(&rm_gu, p, gu, 2) || !raw_maps<FMT>(&rm_dn, p, dn, 1))
        return MOE_ERR_CUDA;
    tc_gateup_kernel<FMT><<<grid, kTcThreads, gu_smem<FMT>(), stream>>>(p, map_x, rm_gu);
    tc_down_kernel<FMT><<<grid, kTcThreads, dn_smem<FMT>(), stream>>>(p, map_h, rm_dn);
    return launch_status();
}

}  // namespace

// Launch the two grouped GEMMs; h is fp16 [T*k][f] inside the caller's workspace.
moe_status tc05_ffn(int fmt, const moe_qpool *W, const int32_t *slot_of, const uint16_t *x, int T, int d, int f, int E,
                    int k, const int32_t *offsets, const int32_t *sorted_tok, const int32_t *sorted_j,
                    const int32_t *active, const float *topk_w, float *out, void *ws, int32_t *dev_status,
                    cudaStream_t stream) {
    return fmt == 2 ? tc05_ffn_fmt<2>(W, slot_of, x, T, d, f, E, k, offsets, sorted_tok, sorted_j, active, topk_w, out,
                                      ws, dev_status, stream)
                    : tc05_ffn_fmt<3>(W, slot_of, x, T, d, f, E, k, offsets, sorted_tok, sorted_j, active, topk_w, out,
                                      ws, dev_status, stream);
}

}  // namespace moe

#ifdef MOE_TC_TRACE
// Copies the wait accounting of the last tensor-core calls (uint64
// [2 kernels][256 CTAs][4 roles][8]) to host memory and clears it.
MOE_API int moe_tc_trace_read(unsigned long long *host) {
    constexpr size_t kWords = size_t(2) * moe::kTraceCtas * 4 * 8;
    static unsigned long long zeros[kWords];
    if (cudaMemcpyFromSymbol(host, moe::g_tc_trace, kWords * 8) != cudaSuccess) return -1;
    if (cudaMemcpyToSymbol(moe::g_tc_trace, zeros, kWords * 8) != cudaSuccess) return -1;
    return 0;
}
#endif
