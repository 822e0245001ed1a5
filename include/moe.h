/*
 * moe.h -- C ABI of libmoe, a CUDA (sm_100a) library for one sparse
 * mixture-of-experts FFN layer with 2-bit / 3-bit block-quantised experts.
 *
 * The layer follows the MoE block described in
 *   [SAITO] "个人开发者用 AI 十天写出 Strata 引擎，让 12GB 显存跑起 1250 亿参数的
 *           Qwen 3.8 Flash Next" (attain.fans repost of an X article),
 *   [JDSSL] "5070ti16g单卡跑qwen 3.8 flash next 新方案最高90t/s Hermes调用60t/s",
 *   [EN]    "Running Qwen3.8-Flash-Next on a 12GB GPU: Custom Engine Hits 65 tok/s":
 * per token a router picks 10 of the layer's 512 experts and one shared expert
 * always runs ([SAITO] section "1250 亿参数，每个词只用得上 2%"); hot experts sit in a
 * GPU-memory cache and the others are computed elsewhere ([JDSSL] section
 * "为什么从 18t/s 变成 60-90t/s"; [SAITO] section "命中率七成，代价是答案会变");
 * weights come in 2-bit and 3-bit tiers ([EN] section "Detailed Performance
 * Numbers"). The pages fix none of the arithmetic; each call below states the
 * definition this library implements.
 *
 * Conventions for every call:
 *  - All array pointers are DEVICE pointers unless a parameter says "host".
 *    The caller allocates and owns every buffer; the library never allocates,
 *    frees or synchronises.
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = the legacy default
 *    stream) and runs asynchronously; results are valid once the stream has
 *    reached that point.
 *  - Host-side checks run first: a null required pointer, a negative or
 *    inconsistent size or an unsupported shape returns an error code at once
 *    and enqueues nothing. T == 0 is valid and enqueues nothing.
 *  - Faults only the device can see (an expert id outside [0,E), a slot
 *    outside the pool, a non-finite logit, too many misses) are OR-ed into
 *    `*dev_status` (MOE_DEV_* bits) and the kernels finish normally; the
 *    caller reads the word after synchronising. `dev_status` may be NULL to
 *    ignore them. Kernels never trap.
 *  - Calls keep no state between invocations and may run concurrently on
 *    different streams with disjoint outputs.
 *  - Shapes: d and f multiples of 256 (d <= 8192, f <= 8192), 1 <= k <= 16,
 *    k <= E <= 4096, T*k < 2^31.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *moe_stream_t; /* same handle as cudaStream_t */

typedef enum moe_status {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1, /* null pointer, negative or inconsistent size   */
    MOE_ERR_UNSUPPORTED = 2, /* shape outside the supported range (see top)   */
    MOE_ERR_WORKSPACE = 3,   /* workspace missing or smaller than required    */
    MOE_ERR_CUDA = 4,        /* a kernel launch was rejected by the runtime   */
    MOE_ERR_OVERFLOW = 5,    /* a size product overflows                     */
    MOE_ERR_HOST = 6         /* host memory or a host thread could not be had */
} moe_status;

/* Device-side status bits, OR-ed into *dev_status. */
#define MOE_DEV_BAD_INDEX 0x1     /* expert id outside [0,E) or repeated in a token */
#define MOE_DEV_BAD_SLOT 0x2      /* slot_of entry outside [-1, num_slots)          */
#define MOE_DEV_NONFINITE 0x4     /* NaN/Inf router logit, or an activation beyond  */
                                  /* the fp16 range used for tensor-core staging    */
#define MOE_DEV_MISS_OVERFLOW 0x8 /* more misses than miss_cap                      */
#define MOE_DEV_TIMEOUT 0x10      /* a bounded in-kernel wait gave up               */

/*
 * Canonical storage of one quantised matrix [R][K] (host or device memory as
 * the call states). K runs along 64-weight blocks.
 *   codes: uint8 [R][K/4]; weight k's 2-bit code (Q2) or low two bits (Q3) at
 *          byte k/4, bits 2*(k%4) and 2*(k%4)+1 (least significant first).
 *   hi:    Q3 only, uint8 [R][K/8]; third code bit of weight k at byte k/8, bit k%8.
 *   scale: fp16 bits [R][K/64], one scale s per block.
 *   min:   Q2 only, fp16 bits [R][K/64], one offset m per block.
 * Q2 weight: w = s*q + m, q in {0..3}.  Q3 weight: w = s*(q-4), q in {0..7}.
 */
typedef struct moe_qmatrix {
    const uint8_t *codes;
    const uint8_t *hi;     /* NULL for Q2 */
    const uint16_t *scale;
    const uint16_t *min;   /* NULL for Q3 */
} moe_qmatrix;

/*
 * A pool of packed experts in device memory: slot s starts at
 * base + s*slot_bytes (256-byte aligned, slot_bytes >= moe_expert_bytes()).
 * Every slot holds one expert (gate [f][d], up [f][d], down [d][f]) in the
 * library's packed record, written by moe_pack_expert. fmt is 2 (Q2) or 3 (Q3).
 */
typedef struct moe_qpool {
    const void *base;
    int64_t slot_bytes;
    int32_t num_slots;
    int32_t fmt;
    int32_t d;
    int32_t f;
} moe_qpool;

/* One routed (token, expert) pair whose expert has no slot in the pool. */
typedef struct moe_miss {
    int32_t layer;
    int32_t expert;
    int32_t token;
    int32_t j;      /* position of the expert in the token's top-k list */
    float gate;     /* its gate weight */
} moe_miss;

/* Human-readable name of a status code (static string, never NULL). */
const char *moe_status_str(moe_status s);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int moe_version(void);

/* ------------------------------------------------------------------ */
/* Packing                                                             */
/* ------------------------------------------------------------------ */

/* Bytes of one packed expert record (a multiple of 256); 0 if the shape is
 * unsupported. Q2 stores 2.5 bits and Q3 3.25 bits per weight, so a
 * d=2048, f=768 expert takes 1,474,560 B (Q2) or 1,916,928 B (Q3). */
size_t moe_expert_bytes(int fmt, int d, int f);

/* Pack one expert from canonical storage (device pointers inside the three
 * host structs) into a record at dst (device, 256-byte aligned,
 * moe_expert_bytes() bytes). The record is a bijective re-ordering of the same
 * bits, arranged for the kernels' loads; its layout is private to the library. */
moe_status moe_pack_expert(int fmt, int d, int f, const moe_qmatrix *gate, const moe_qmatrix *up,
                           const moe_qmatrix *down, void *dst, moe_stream_t stream);

/* Same as moe_pack_expert, on the host: canonical host arrays -> host record. */
moe_status moe_pack_expert_host(int fmt, int d, int f, const moe_qmatrix *gate, const moe_qmatrix *up,
                                const moe_qmatrix *down, void *dst_host);

/* Inverse of moe_pack_expert_host: host record -> canonical host arrays
 * (the struct members point at caller-owned writable host buffers). */
moe_status moe_unpack_expert_host(int fmt, int d, int f, const void *record_host, moe_qmatrix *gate,
                                  moe_qmatrix *up, moe_qmatrix *down);

/* ------------------------------------------------------------------ */
/* The layer's steps                                                   */
/* ------------------------------------------------------------------ */

/*
 * Router and top-k gates ([SAITO] "1250 亿参数，每个词只用得上 2%": 10 of 512
 * experts per token; the router is kept on the GPU per "命中率七成，代价是答案会变").
 *   x       bf16 bits [T][d], row-major
 *   Wr      fp32 [E][d], row-major
 *   bias    fp32 [E] or NULL
 *   logits  fp32 [T][E] (output): the router logit as an fp32 value with a
 *           fixed order of operations -- d is cut into d/128 chunks; inside
 *           chunk i accumulator l (0..31) takes elements 128i+4l+j, j=0..3, by
 *           fused multiply-add, chunks in order; the 32 accumulators are
 *           combined by acc[l] += acc[l^o] for o = 16,8,4,2,1; the bias is
 *           added last. d must be a multiple of 128 (256 for the whole library).
 *   topk_idx int32 [T][k] (output): the k experts that come first in the
 *           order (logit desc, id asc), listed in ascending id.
 *   topk_w  fp32 [T][k] (output): softmax of the k selected logits (equal to
 *           a full softmax renormalised over the selected experts).
 * A NaN logit sets MOE_DEV_NONFINITE and is never selected. x and Wr must be
 * 16-byte aligned (else MOE_ERR_INVALID_ARG).
 */
moe_status moe_route(const uint16_t *x, const float *Wr, const float *bias, int T, int d, int E, int k,
                     float *logits, int32_t *topk_idx, float *topk_w, int32_t *dev_status,
                     moe_stream_t stream);

/* Workspace bytes moe_permute needs for (T, k, E); may be 0. */
size_t moe_permute_workspace_bytes(int T, int k, int E);

/*
 * Token -> expert permutation: the T*k pairs p = t*k + j are sorted by expert
 * id and, within an expert, by p (a stable counting sort).
 *   counts   int32 [E]      pairs per expert
 *   offsets  int32 [E+1]    exclusive prefix sum of counts
 *   sorted_tok, sorted_j int32 [T*k]: pair at sorted position s
 *   inv      int32 [T*k]    inv[p] = sorted position of pair p
 *   active   int32 [E+1]    active[0] = number of experts with >= 1 pair,
 *                           active[1..] = those expert ids, ascending
 *   ws       workspace of moe_permute_workspace_bytes() bytes (may be NULL if 0)
 * Ids outside [0,E) or repeated within a token set MOE_DEV_BAD_INDEX.
 */
moe_status moe_permute(const int32_t *topk_idx, int T, int k, int E, int32_t *counts, int32_t *offsets,
                       int32_t *sorted_tok, int32_t *sorted_j, int32_t *inv, int32_t *active, void *ws,
                       size_t ws_bytes, int32_t *dev_status, moe_stream_t stream);

/*
 * Expert-cache lookup ([JDSSL] "为什么从 18t/s 变成 60-90t/s": a GPU-memory cache of
 * hot experts; [SAITO] "命中率七成，代价是答案会变": experts outside it are computed
 * on the CPU). Runs after moe_permute on the same routing.
 *   slot_of      int32 [E]: HBM slot of each expert of this layer, -1 = not resident
 *   num_slots    slots in the pool (entries >= num_slots set MOE_DEV_BAD_SLOT
 *                and are treated as misses)
 *   slot_of_pair int32 [T*k] (output): slot_of[topk_idx[p]] for pair p (-1 = miss)
 *   miss         moe_miss [miss_cap] (output): every pair whose expert is not
 *                resident, ordered by (expert, token); entries past miss_cap are
 *                dropped and set MOE_DEV_MISS_OVERFLOW
 *   miss_count   int32 [1] (output): the true number of misses
 *   expert_counts int32 [E] or NULL: every routed pair (hit or miss) adds 1
 *                to its expert's entry (atomically; the caller zeroes it when
 *                a counting window starts) -- the use counts the cache policy
 *                reads in bulk (moe_cache_policy_observe_counts)
 */
moe_status moe_cache_lookup(const int32_t *slot_of, int32_t num_slots, int32_t layer, const int32_t *topk_idx,
                            const float *topk_w, const int32_t *offsets, const int32_t *sorted_tok,
                            const int32_t *sorted_j, int T, int k, int E, int32_t *slot_of_pair, moe_miss *miss,
                            int32_t *miss_count, int32_t miss_cap, int32_t *expert_counts, int32_t *dev_status,
                            moe_stream_t stream);

/* Workspace bytes moe_expert_ffn_q2/q3 need for (T, k, d, f). With T*k < 512
 * only the weight-streaming path can run and the workspace is h as fp32,
 * T*k*f*4 bytes. With T*k >= 512 the tensor-core path may run, and the size is
 * the larger of that and T*k*f fp16 (h, rounded up to 256 B) + T*k*d fp16
 * (activation rows in sorted order). */
size_t moe_expert_ffn_workspace_bytes(int T, int k, int d, int f);

/*
 * SwiGLU experts on the packed pool: for every active expert e that has a slot
 * and every sorted pair s of e (token t = sorted_tok[s]):
 *     a = Wg_e x_t,  u = Wu_e x_t,  h = silu(a) * u = a / (1 + exp(-a)) * u,
 *     y_e = Wd_e h.
 *   W        host pointer to the pool description (W->fmt must match the call)
 *   slot_of  int32 [E]: slot of each expert, -1 = skip (a miss)
 *   x        bf16 bits [T][d]
 *   offsets, sorted_tok, sorted_j, active: from moe_permute
 *   topk_w   NULL: out is y_perm fp32 [T*k][d], row s = y_e for pair s (rows of
 *            skipped experts are left untouched);
 *            non-NULL: out is y fp32 [T][d] and receives y[t] += topk_w[t*k+j] * y_e
 *            (atomic adds; the caller initialises y).
 * The shared expert is the case E = 1, k = 1, offsets = {0, T},
 * sorted_tok[t] = t, sorted_j[t] = 0, active = {1, 0}, slot_of = {its slot}.
 * Activations are staged as fp16 for the tensor cores; |x| or |h| beyond
 * 65504 sets MOE_DEV_NONFINITE.
 * Paths: with T*k < 512 a weight-streaming kernel reads each expert's packed
 * codes once per 8 tokens (mma.sync fragments built from the codes); with
 * T*k >= 512 and E <= 1024 (prefill) both calls run grouped GEMMs on the
 * tcgen05 tensor cores, dequantising each 128-row weight tile to fp16 in
 * registers and storing it to tensor memory (one fp16 rounding of
 * w = s*q + m (Q2, one fused multiply-add) or w = s*(q-4) (Q3));
 * the workspace then holds h as fp16 [T*k][f]
 * followed by the activation rows in sorted pair order as fp16 [T*k][d]; ws
 * must then be 256-byte and x 16-byte aligned (else MOE_ERR_INVALID_ARG).
 * A pool may hold records of both formats (slot_bytes >= the larger record):
 * give each call a slot table in which the other format's experts are -1.
 */
moe_status moe_expert_ffn_q2(const moe_qpool *W, const int32_t *slot_of, const uint16_t *x, int T, int d, int f,
                             int E, int k, const int32_t *offsets, const int32_t *sorted_tok, const int32_t *sorted_j,
                             const int32_t *active, const float *topk_w, float *out, void *ws, size_t ws_bytes,
                             int32_t *dev_status, moe_stream_t stream);
moe_status moe_expert_ffn_q3(const moe_qpool *W, const int32_t *slot_of, const uint16_t *x, int T, int d, int f,
                             int E, int k, const int32_t *offsets, const int32_t *sorted_tok, const int32_t *sorted_j,
                             const int32_t *active, const float *topk_w, float *out, void *ws, size_t ws_bytes,
                             int32_t *dev_status, moe_stream_t stream);

/*
 * Host completion of the miss list: the experts that have no GPU slot are
 * computed on the host, as the engine of "5070ti16g单卡跑qwen 3.8 flash next
 * 新方案最高90t/s Hermes 调用60t/s" (section "为什么从 18t/s 变成 60-90t/s") does
 * with the experts kept in system RAM. For every record i of miss[0..n):
 *   y[miss[i].token] += miss[i].gate * down(silu(gate_proj x) * up_proj x),
 * x = x[miss[i].token], in fp32 from the expert's canonical storage (w = s*q+m
 * or s*(q-4) applied per 64-block to the block's code-weighted sum, that sum
 * formed from 16 per-byte-position partial sums added in a fixed order).
 * Results are added in record order, so y does not depend on nthreads.
 *   fmt, d, f  format and shapes (as for the pool)
 *   experts    moe_qmatrix [E][3] (host): gate [f][d], up [f][d], down [d][f]
 *              of every expert of this layer in canonical host storage; only
 *              the experts the records name are read
 *   miss, n    the layer's miss records (host), as moe_cache_lookup or
 *              moe_layer_decode wrote them; every record must name `layer`
 *   x          bf16 bits [T][d] (host), the layer's input
 *   y          fp32 [T][d] (host), accumulated into (e.g. the GPU's partial y)
 *   nthreads   worker threads (0 = the machine's hardware threads)
 * Returns MOE_ERR_INVALID_ARG, before any change to y, for a record with
 * another layer, an expert outside [0, E), a token outside [0, T) or an expert
 * whose matrices are missing (NULL codes/scale, min for Q2, hi for Q3), and
 * MOE_ERR_HOST, with y unchanged, if host memory for the per-record results
 * cannot be had. If fewer threads than asked can be started, the call finishes
 * the work on those it has.
 * Blocking; no GPU involvement.
 */
moe_status moe_complete_misses_host(int fmt, int d, int f, const moe_qmatrix *experts, int E, const moe_miss *miss,
                                    int32_t n, int32_t layer, const uint16_t *x, int T, float *y, int nthreads);

/*
 * Miss engine: a pool of host worker threads that completes miss lists as the
 * GPU publishes them, so that the host works on one layer's misses while the
 * GPU runs the next layers ([SAITO] "命中率七成，代价是答案会变": the CPU computes
 * the experts that are not in GPU memory during the same round as the GPU).
 *   create   nthreads workers (0 = the machine's hardware threads);
 *            MOE_ERR_HOST if threads or memory cannot be had
 *   submit   queue one layer: the arguments of moe_complete_misses_host, with
 *            the record count read from *count (host memory) once it is >= 0
 *            (at most miss_cap records are used). A miss list and count that
 *            moe_layer_decode / moe_stack_decode write to mapped pinned host
 *            memory are published in that order (the count last, after a
 *            system-wide fence): set *count to -1 before the launch and submit
 *            at once. All pointers must stay valid until wait returns. A count
 *            still negative after 10 s fails the job with MOE_ERR_HOST.
 *            Jobs run in any order and concurrently; each job adds its records
 *            into its y in record order (y independent of the thread count).
 *   wait     block until every submitted job has finished; returns the first
 *            error among them (MOE_OK if none) and forgets them
 *   destroy  wait, then stop the workers
 * One thread at a time may call submit/wait on an engine.
 */
typedef struct moe_miss_engine moe_miss_engine;
moe_status moe_miss_engine_create(int nthreads, moe_miss_engine **engine);
moe_status moe_miss_engine_submit(moe_miss_engine *engine, int fmt, int d, int f, const moe_qmatrix *experts, int E,
                                  const moe_miss *miss, const int32_t *count, int32_t miss_cap, int32_t layer,
                                  const uint16_t *x, int T, float *y);
moe_status moe_miss_engine_wait(moe_miss_engine *engine);
void moe_miss_engine_destroy(moe_miss_engine *engine);

/*
 * Expert-cache policy ([SAITO] "命中率七成，代价是答案会变": the free GPU room is
 * filled with the most frequently called experts, swapped while the
 * conversation runs). Host state in caller-owned memory; integer arithmetic,
 * so decisions are exactly reproducible:
 *   - observe: every routed pair of `layer` adds 1 to count[layer][expert];
 *     every `epoch` tokens (counted on layer 0) all counts are halved;
 *   - plan: free slots go to the non-resident (layer, expert) with the highest
 *     counts (> 0); then the best non-resident replaces the worst resident
 *     while best.count > worst.count + margin; at most max_swaps changes.
 *     Candidates rank by count desc, then layer*E+expert asc; victims by count
 *     asc, then layer*E+expert desc; free slots are filled in ascending order.
 * The slot pool is shared by all L layers: slot_of is int32 [L][E] (host),
 * -1 = not resident, each slot in [0, S) held at most once; plan updates it in
 * place and lists the changes. The caller then copies every admitted expert's
 * record into its slot and the slot table to the device.
 */
typedef struct moe_swap {
    int32_t slot;
    int32_t layer_in, expert_in;    /* the expert that now holds the slot      */
    int32_t layer_out, expert_out;  /* its previous holder, -1/-1 if it was free */
} moe_swap;

/* Bytes of policy state for L layers of E experts (0 if unsupported). */
size_t moe_cache_policy_bytes(int L, int E);

/* Initialise the state (all counts 0); S slots; epoch > 0 tokens; margin >= 0. */
moe_status moe_cache_policy_init(void *state, size_t bytes, int L, int E, int S, int epoch, int margin);

/* Count one layer call's routing: topk_idx int32 [T][k] (host). */
moe_status moe_cache_policy_observe(void *state, int layer, const int32_t *topk_idx, int T, int k);

/* Count a window of `tokens` token steps at once from per-expert counts
 * (host int32 [L][E], e.g. a copy of the device counters that
 * moe_cache_lookup / moe_layer_decode / moe_stack_decode add to): the token
 * clock advances by `tokens` first (halving all counts once per full epoch),
 * then every count is added. For a window of one token step through all
 * layers this equals moe_cache_policy_observe on each layer in order. */
moe_status moe_cache_policy_observe_counts(void *state, const int32_t *counts_host, int tokens);

/* Plan slot changes; returns the number written to swaps (<= max_swaps), or
 * -(moe_status) on an invalid state or slot table (slot_of then unchanged). */
int32_t moe_cache_policy_plan(void *state, int32_t *slot_of, moe_swap *swaps, int32_t max_swaps);

/*
 * Diagnostic for the bounded waits: one CTA runs the library's two in-kernel
 * waits against objects that nothing completes -- the device counter *counter
 * (read with acquire loads) awaited until >= target, then a fresh shared-memory
 * mbarrier phase with no arrival. Each gives up after the library's wait limit
 * (100 ms, or a poll count that bounds it should the timer stand still) and
 * sets MOE_DEV_TIMEOUT in *dev_status; elapsed_ns (device, uint64 [2]) receives
 * the two durations. With *counter >= target the first wait returns at once.
 * All pointers are device pointers; asynchronous on the stream.
 */
moe_status moe_debug_wait_probe(const uint32_t *counter, uint32_t target, uint64_t *elapsed_ns,
                                int32_t *dev_status, moe_stream_t stream);

/* Workspace bytes moe_layer_decode and moe_stack_decode need for (T, k, f, E):
 * two grid counters and 2 x 8 fp32 [T][E] logit buffers (the logits are
 * written in 8 copies, which the launch's CTAs read in turn). */
size_t moe_layer_decode_workspace_bytes(int T, int k, int f, int E);
size_t moe_stack_decode_workspace_bytes(int T, int k, int f, int E);

/*
 * The whole layer for a few tokens (decode, or an MTP verify batch of one token
 * plus drafts -- [SAITO] "命中率七成，代价是答案会变" verifies three drafts at once) in
 * one cooperative launch of thread-block clusters: router + top-k gates,
 * permutation, cache lookup, routed experts, shared expert and gate-weighted
 * combine, as defined by moe_route, moe_permute, moe_cache_lookup,
 * moe_expert_ffn_q2/q3 and moe_combine. Routing, permutation, slots and misses
 * are identical to those calls; y agrees with them up to the order of its fp32
 * additions (each expert's hidden activations are formed from C partial sums
 * over slices of d added in a fixed order, and the experts' contributions are
 * added into y with atomics).
 *   W, slot_of   pool and this layer's expert -> slot table (W->fmt 2 or 3)
 *   shared_slot  pool slot of the layer's shared expert
 *   layer        copied into miss records
 *   x, Wr, bias  as moe_route; T <= 8, E <= 512, d <= 2048, f <= 4096;
 *                x, Wr and y 16-byte aligned
 *   logits .. miss_count  outputs of the step-by-step calls, each may be NULL
 *   expert_counts int32 [E] or NULL: routed pairs added per expert, as for
 *                moe_cache_lookup
 *   y            fp32 [T][d] (output, overwritten)
 *   ws           moe_layer_decode_workspace_bytes() bytes, 256-byte aligned,
 *                zero-filled before first use; each launch leaves its counters
 *                zeroed again (zero it again after a MOE_DEV_TIMEOUT)
 * The launch uses every SM (one CTA per SM, clusters of 4 CTAs when d is a
 * multiple of 1024, of 2 when a multiple of 512, else of 1); two launches on
 * different streams must not share a workspace, and launches that would run
 * at the same time as other work on the GPU wait for SMs (the grid must be
 * co-resident; a grid-wide wait that gives up sets MOE_DEV_TIMEOUT).
 */
moe_status moe_layer_decode(const moe_qpool *W, const int32_t *slot_of, int32_t shared_slot, int32_t layer,
                            const uint16_t *x, const float *Wr, const float *bias, int T, int d, int f, int E, int k,
                            float *logits, int32_t *topk_idx, float *topk_w, int32_t *counts, int32_t *offsets,
                            int32_t *sorted_tok, int32_t *sorted_j, int32_t *inv, int32_t *active,
                            int32_t *slot_of_pair, moe_miss *miss, int32_t *miss_count, int32_t miss_cap,
                            int32_t *expert_counts, float *y, void *ws, size_t ws_bytes, int32_t *dev_status,
                            moe_stream_t stream);

/*
 * L layers of moe_layer_decode in one launch, in order: layer l + 1 starts
 * once every contribution to layer l's y is in place (a grid barrier), so its
 * input could have been derived from layer l's output; while layer l's experts
 * stream, every CTA asks the L2 for its slice of layer l + 1's router rows and
 * shared expert (weights that do not depend on routing). The ([SAITO]
 * "1250 亿参数，每个词只用得上 2%") model has 48 such layers.
 *   W            one pool holding every layer's resident experts
 *   slot_of      int32 [L][E]: each layer's expert -> slot table (-1 = miss)
 *   shared_slot  int32 [L] (device): each layer's shared-expert slot
 *   layer0       layer id of the first layer (miss records carry layer0 + l)
 *   x            bf16 [L][T][d]: each layer's input
 *   Wr, bias     fp32 [L][E][d], [L][E] (bias may be NULL)
 *   topk_idx, topk_w, slot_of_pair  [L][T*k] outputs as moe_layer_decode (may be NULL)
 *   miss         moe_miss [L][miss_cap], miss_count int32 [L] (may be NULL);
 *                layer l's records and then its count are written as the
 *                layer ends (the count after a system-wide fence), so they may
 *                live in mapped pinned host memory read while the launch runs
 *   expert_counts int32 [L][E] or NULL: routed pairs added per (layer, expert)
 *   y            fp32 [L][T][d] (output)
 *   ws           moe_stack_decode_workspace_bytes() bytes, as moe_layer_decode
 * Shapes and limits as moe_layer_decode.
 */
moe_status moe_stack_decode(const moe_qpool *W, int L, const int32_t *slot_of, const int32_t *shared_slot,
                            int32_t layer0, const uint16_t *x, const float *Wr, const float *bias, int T, int d, int f,
                            int E, int k, int32_t *topk_idx, float *topk_w, int32_t *slot_of_pair, moe_miss *miss,
                            int32_t *miss_count, int32_t miss_cap, int32_t *expert_counts, float *y, void *ws,
                            size_t ws_bytes, int32_t *dev_status, moe_stream_t stream);

/*
 * moe_expert_ffn_q2 without a caller-supplied workspace. The pages have no
 * counterpart to this call; it exists for callers that cannot allocate device
 * memory -- for example a plugin inside a host framework that owns every device
 * buffer and hands the plugin only its inputs and outputs, or a serving loop
 * that allocates nothing after start-up so its memory footprint is fixed and no
 * request can fail on an out-of-memory error. Arguments and results are those of
 * moe_expert_ffn_q2; the caller still passes every input and output.
 *   Scratch: the workspace moe_expert_ffn_q2 would need (hidden activations,
 *   plus an fp16 copy of x on the tensor-core path) goes to one 4 MiB array
 *   built into the library; each GPU that loads the library holds its own copy
 *   until the process exits. moe_expert_ffn_workspace_bytes(T, k, d, f) > 4 MiB
 *   returns MOE_ERR_WORKSPACE before anything is enqueued. For d = 2048,
 *   f = 768 that admits T*k <= 744: below 512 pairs the scratch holds
 *   T*k*f*4 bytes of h; from 512 pairs on the tensor-core layout needs
 *   T*k*(2f + 2d) bytes (5,632 per pair), and 744 * 5,632 <= 4 MiB < 745 * 5,632.
 *   Set-up: the first call on a device looks up that device's copy of the
 *   array (cudaGetSymbolAddress, with the device current); make that first call
 *   before any stream capture. The address is kept per device and driver
 *   context and looked up again when a call runs in a context it has not seen
 *   (for example after cudaDeviceReset). Lookup failures return MOE_ERR_CUDA.
 *   Sharing: every call on a device uses the same array, which keeps whatever
 *   the last call wrote (nothing in it needs to start at zero: each call writes
 *   every entry it reads). Calls that can overlap on the GPU -- on different
 *   streams without ordering between them -- race on the array and corrupt each
 *   other's results; order them on one stream or use moe_expert_ffn_q2.
 *   It calls no cudaMalloc, cudaFree or other allocating routine.
 */
moe_status moe_expert_ffn_q2_noalloc(const moe_qpool *W, const int32_t *slot_of, const uint16_t *x, int T, int d,
                                     int f, int E, int k, const int32_t *offsets, const int32_t *sorted_tok,
                                     const int32_t *sorted_j, const int32_t *active, const float *topk_w, float *out,
                                     int32_t *dev_status, moe_stream_t stream);

/*
 * Gate-weighted combine plus the shared expert:
 *   y[t] = y_shared[t] + sum_{j=0..k-1, slot_of_pair[t*k+j] >= 0} topk_w[t*k+j] * y_perm[inv[t*k+j]]
 *   y_perm fp32 [T*k][d]; inv, topk_w, slot_of_pair [T*k] (slot_of_pair may be
 *   NULL = every pair resident); y_shared fp32 [T][d] or NULL (= 0); y fp32 [T][d].
 */
moe_status moe_combine(const float *y_perm, const int32_t *inv, const float *topk_w, const int32_t *slot_of_pair,
                       const float *y_shared, int T, int k, int d, float *y, moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H */
