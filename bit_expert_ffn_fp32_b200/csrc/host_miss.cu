// Host completion of the miss list.
//
// Experts that have no slot in the GPU pool are not computed on the GPU: the
// lookup step lists them as (layer, expert, token, j, gate) records, and the
// host computes them, as the engine of "5070ti16g单卡跑qwen 3.8 flash next
// 新方案最高90t/s Hermes 调用60t/s" (section "为什么从 18t/s 变成 60-90t/s") does
// with the experts that stay in system RAM, while the GPU runs the rest of the
// model ("个人开发者用 AI 十天写出 Strata 引擎，让 12GB 显存跑起 1250 亿参数的 Qwen
// 3.8 Flash Next", section "命中率七成，代价是答案会变": the CPU and the GPU each wait
// part of a round for the other). This file is that host step: for every
// record, y[token] += gate * down(silu(gate_proj x) * up_proj x), the expert's
// weights read from their canonical storage in host memory.
//
// Dot products: a 64-weight block's code-weighted sum sum_k q_k v_k is formed
// from the input vector stored bit-position major -- lo[i][j] = v[4j + i], the
// input of the 2-bit field at bits 2i..2i+1 of code byte j -- so that for each
// field position i the 16 code bytes are shifted, masked, converted and
// multiplied with 16 contiguous inputs (loops the compiler vectorises, with
// one accumulator per byte position, summed in a fixed order); Q3 adds 4 x the
// high-bit plane the same way (hi[i][j] = v[8j + i]). The block's scale and
// min are applied to its sum:
//   sum_k w_k v_k = s * sum_k q_k v_k + m * sum_k v_k        (Q2, w = s*q + m)
//                 = s * (sum_k q_k v_k - 4 * sum_k v_k)      (Q3, w = s*(q-4)).
// Work is spread over threads one expert at a time; the per-record results are
// added into y in record order, so y does not depend on the thread count.
//
// Two entry points: moe_complete_misses_host (blocking, one layer) and a miss
// engine (a pool of worker threads) that takes layers as they are published:
// a submitted layer waits for its record count to become >= 0 -- the decode
// kernels write the records and then the count, after a system-scope fence,
// so the host sees a layer's misses while the GPU is still on later layers.
#include <algorithm>
#include <atomic>
#include <chrono>
#include <cmath>
#include <condition_variable>
#include <cstring>
#include <deque>
#include <memory>
#include <mutex>
#include <thread>
#include <vector>

#include "common.cuh"

namespace moe {
namespace {

// IEEE binary16 bits -> float (exact): subnormals m*2^-24, normals (1024+m)*2^(e-25).
float half_value(uint16_t h) {
    const int e = (h >> 10) & 0x1f;
    const int m = h & 0x3ff;
    float v;
    if (e == 0)
        v = std::ldexp(float(m), -24);
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = std::ldexp(float(m | 0x400), e - 25);
    return (h & 0x8000) ? -v : v;
}

// every fp16 bit pattern's value, built once
const std::vector<float> &half_table() {
    static const std::vector<float> t = [] {
        std::vector<float> v(65536);
        for (int i = 0; i < 65536; ++i) v[i] = half_value(uint16_t(i));
        return v;
    }();
    return t;
}

float bf16_value(uint16_t b) {
    const uint32_t u = uint32_t(b) << 16;
    float v;
    std::memcpy(&v, &u, 4);
    return v;
}

// One input vector v[K] stored for the block dot products (see the top of the file).
struct PermInput {
    std::vector<float> lo;    // [K/64][4][16]: v[64b + 4j + i] at [b][i][j]
    std::vector<float> hi;    // [K/64][8][8]:  v[64b + 8j + i] at [b][i][j] (Q3)
    std::vector<float> bsum;  // [K/64]: block sums of v

    void build(const float *v, int K, bool q3) {
        const int NB = K / 64;
        lo.resize(size_t(NB) * 64);
        for (int b = 0; b < NB; ++b)
            for (int i = 0; i < 4; ++i)
                for (int j = 0; j < 16; ++j) lo[size_t(b) * 64 + i * 16 + j] = v[64 * b + 4 * j + i];
        if (q3) {
            hi.resize(size_t(NB) * 64);
            for (int b = 0; b < NB; ++b)
                for (int i = 0; i < 8; ++i)
                    for (int j = 0; j < 8; ++j) hi[size_t(b) * 64 + i * 8 + j] = v[64 * b + 8 * j + i];
        }
        bsum.assign(NB, 0.f);
        for (int b = 0; b < NB; ++b) {
            float p[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            for (int k = 0; k < 64; k += 8)
                for (int j = 0; j < 8; ++j) p[j] += v[64 * b + k + j];
            bsum[b] = ((p[0] + p[1]) + (p[2] + p[3])) + ((p[4] + p[5]) + (p[6] + p[7]));
        }
    }
};

}  // namespace

// Rows r0 .. r1-1 of a canonical matrix [R][K] against one input: out[r - r0].
// Built for AVX-512, AVX2 and plain x86-64; the loader picks one at run time.
__attribute__((target_clones("avx512f", "avx2", "default"), noinline)) void moe_host_rows_dot(
    const uint8_t *codes, const uint8_t *hibits, const uint16_t *scale, const uint16_t *mn, int q3, int K, int r0,
    int r1, const float *lo, const float *hi, const float *bsum, const float *hv, float *out) {
    const int NB = K / 64;
    for (int r = r0; r < r1; ++r) {
        const uint8_t *c = codes + size_t(r) * (K / 4);
        const uint8_t *h = q3 ? hibits + size_t(r) * (K / 8) : nullptr;
        const uint16_t *sc = scale + size_t(r) * NB;
        const uint16_t *mi = q3 ? nullptr : mn + size_t(r) * NB;
        float acc = 0.f;
        for (int b = 0; b < NB; ++b) {
            const uint8_t *cb = c + 16 * b;
            const float *lb = lo + size_t(b) * 64;
            float part[16];
            for (int j = 0; j < 16; ++j) part[j] = 0.f;
            for (int i = 0; i < 4; ++i)
                for (int j = 0; j < 16; ++j) part[j] += float((cb[j] >> (2 * i)) & 3) * lb[i * 16 + j];
            float q = 0.f;
            for (int j = 0; j < 16; j += 4) q += (part[j] + part[j + 1]) + (part[j + 2] + part[j + 3]);
            const float s = hv[sc[b]];
            if (!q3) {
                acc += s * q + hv[mi[b]] * bsum[b];
            } else {
                const uint8_t *hb = h + 8 * b;
                const float *hbv = hi + size_t(b) * 64;
                // 16 lanes: lane l takes bit 2ii + l/8 of byte l%8 (weight 8(l%8) + 2ii + l/8),
                // whose permuted input sits at hbv[16 ii + l]
                uint32_t hw[16];
                for (int l = 0; l < 16; ++l) hw[l] = uint32_t(hb[l & 7]) >> (l >> 3);
                float hp[16];
                for (int l = 0; l < 16; ++l) hp[l] = 0.f;
                for (int ii = 0; ii < 4; ++ii)
                    for (int l = 0; l < 16; ++l) hp[l] += float((hw[l] >> (2 * ii)) & 1u) * hbv[16 * ii + l];
                float hq = 0.f;
                for (int l = 0; l < 16; l += 4) hq += (hp[l] + hp[l + 1]) + (hp[l + 2] + hp[l + 3]);
                acc += s * ((q + 4.0f * hq) - 4.0f * bsum[b]);
            }
        }
        out[r - r0] = acc;
    }
}

namespace {

void matrix_dot(const moe_qmatrix &m, int fmt, int K, int R, const PermInput &in, float *out) {
    moe_host_rows_dot(m.codes, m.hi, m.scale, m.min, fmt == 3, K, 0, R, in.lo.data(),
                      fmt == 3 ? in.hi.data() : nullptr, in.bsum.data(), half_table().data(), out);
}

bool matrix_ok(const moe_qmatrix &m, int fmt) {
    return m.codes && m.scale && (fmt == 2 ? m.min != nullptr : m.hi != nullptr);
}

// Work buffers of one thread.
struct Scratch {
    PermInput in;
    std::vector<float> xf, a, u, h;
};

// One expert's FFN for one record: out[d] = down(silu(gate x) * up x) (no gate weight).
void expert_record(const moe_qmatrix *q, int fmt, int d, int f, const uint16_t *xrow, Scratch &w, float *out) {
    w.xf.resize(d);
    w.a.resize(f);
    w.u.resize(f);
    w.h.resize(f);
    for (int k = 0; k < d; ++k) w.xf[k] = bf16_value(xrow[k]);
    w.in.build(w.xf.data(), d, fmt == 3);
    matrix_dot(q[0], fmt, d, f, w.in, w.a.data());
    matrix_dot(q[1], fmt, d, f, w.in, w.u.data());
    for (int r = 0; r < f; ++r) w.h[r] = w.a[r] / (1.0f + std::exp(-w.a[r])) * w.u[r];
    w.in.build(w.h.data(), f, fmt == 3);
    matrix_dot(q[2], fmt, f, d, w.in, out);
}

// Records checked before any work: this layer, an expert and token in range,
// the expert's matrices given.
moe_status check_records(int fmt, const moe_qmatrix *experts, int E, const moe_miss *miss, int32_t n, int32_t layer,
                         int T) {
    for (int32_t i = 0; i < n; ++i) {
        const moe_miss &m = miss[i];
        if (m.layer != layer || m.expert < 0 || m.expert >= E || m.token < 0 || m.token >= T)
            return MOE_ERR_INVALID_ARG;
        const moe_qmatrix *q = experts + size_t(m.expert) * 3;
        if (!matrix_ok(q[0], fmt) || !matrix_ok(q[1], fmt) || !matrix_ok(q[2], fmt)) return MOE_ERR_INVALID_ARG;
    }
    return MOE_OK;
}

// Records grouped by expert (stable: record order kept inside a group).
void group_records(const moe_miss *miss, int32_t n, std::vector<int32_t> &order, std::vector<int32_t> &begin) {
    order.resize(n);
    for (int32_t i = 0; i < n; ++i) order[i] = i;
    std::stable_sort(order.begin(), order.end(), [&](int32_t a, int32_t b) { return miss[a].expert < miss[b].expert; });
    begin.clear();
    for (int32_t i = 0; i < n; ++i)
        if (i == 0 || miss[order[i]].expert != miss[order[i - 1]].expert) begin.push_back(i);
    begin.push_back(n);
}

// y[token] += gate * contrib[record], in record order.
void accumulate(const moe_miss *miss, int32_t n, int d, const float *contrib, float *y) {
    for (int32_t i = 0; i < n; ++i) {
        float *yr = y + size_t(miss[i].token) * d;
        const float g = miss[i].gate;
        const float *c = contrib + size_t(i) * d;
        for (int k = 0; k < d; ++k) yr[k] += g * c[k];
    }
}

// The validated work of moe_complete_misses_host. May throw (std::bad_alloc,
// std::system_error) before y is touched; y is written only at the end.
moe_status complete_misses(int fmt, int d, int f, const moe_qmatrix *experts, const moe_miss *miss, int32_t n,
                           const uint16_t *x, float *y, int nthreads) {
    std::vector<int32_t> order, group_begin;
    group_records(miss, n, order, group_begin);
    const int ngroups = int(group_begin.size()) - 1;
    std::vector<float> contrib(size_t(n) * d);  // FFN output of record i (without its gate)
    std::atomic<int> next_group{0};
    std::atomic<bool> failed{false};
    auto work = [&]() {
        Scratch w;
        while (true) {
            const int gi = next_group.fetch_add(1);
            if (gi >= ngroups) break;
            const moe_qmatrix *q = experts + size_t(miss[order[group_begin[gi]]].expert) * 3;
            for (int g = group_begin[gi]; g < group_begin[gi + 1]; ++g) {  // one token at a time
                const int rec = order[g];
                expert_record(q, fmt, d, f, x + size_t(miss[rec].token) * d, w, &contrib[size_t(rec) * d]);
            }
        }
    };
    auto worker = [&]() {
        try {
            work();
        } catch (...) {
            failed = true;
            next_group = ngroups;  // the other workers stop at their next group
        }
    };
    const int hw = int(std::max(1u, std::thread::hardware_concurrency()));
    const int nth = std::max(1, std::min(nthreads > 0 ? nthreads : hw, ngroups));
    std::vector<std::thread> pool;
    pool.reserve(nth);
    try {
        for (int t = 1; t < nth; ++t) pool.emplace_back(worker);
    } catch (...) {  // fewer threads than asked: the started ones and this one finish the work
    }
    worker();
    for (auto &th : pool) th.join();
    if (failed) return MOE_ERR_HOST;
    accumulate(miss, n, d, contrib.data(), y);
    return MOE_OK;
}

}  // namespace

// ---------------------------------------------------------------- miss engine
// A submitted layer is a job; once its count is published the job is split
// into one task per missed expert, and the worker that finishes its last task
// adds the results into y in record order.
struct MissJob {
    int fmt, d, f, E, T;
    const moe_qmatrix *experts;
    const moe_miss *miss;
    const volatile int32_t *count;
    int32_t cap, layer;
    const uint16_t *x;
    float *y;
    // filled when the count is seen
    int32_t n = 0;
    std::vector<int32_t> order, begin;
    std::vector<float> contrib;
    std::atomic<int> left{0};  // expert tasks not finished
    std::atomic<bool> failed{false};
};

struct MissTask {
    MissJob *job;
    int group;  // -1: wait for the count and split the job
};

}  // namespace moe

struct moe_miss_engine {
    std::mutex mu;
    std::condition_variable cv_work, cv_done;
    std::deque<moe::MissTask> tasks;
    std::vector<std::unique_ptr<moe::MissJob>> jobs;
    int pending = 0;  // jobs not finished
    bool stop = false;
    moe_status first_error = MOE_OK;
    std::vector<std::thread> workers;
};

namespace moe {
namespace {

constexpr double kCountWaitS = 10.0;  // a count still unpublished after this fails the job

void finish_job(moe_miss_engine *eng, moe_status st) {
    std::lock_guard<std::mutex> lock(eng->mu);
    if (st != MOE_OK && eng->first_error == MOE_OK) eng->first_error = st;
    if (--eng->pending == 0) eng->cv_done.notify_all();
}

// Wait for the job's count, check and group its records, queue its expert tasks.
void start_job(moe_miss_engine *eng, MissJob *job) {
    const auto t0 = std::chrono::steady_clock::now();
    int32_t n = job->count ? *job->count : job->cap;
    while (n < 0) {
        if (std::chrono::duration<double>(std::chrono::steady_clock::now() - t0).count() > kCountWaitS) {
            finish_job(eng, MOE_ERR_HOST);
            return;
        }
        std::this_thread::yield();
        n = *job->count;
    }
    std::atomic_thread_fence(std::memory_order_acquire);
    n = std::min(n, job->cap);
    const moe_status st = check_records(job->fmt, job->experts, job->E, job->miss, n, job->layer, job->T);
    if (st != MOE_OK || n == 0) {
        finish_job(eng, st);
        return;
    }
    job->n = n;
    group_records(job->miss, n, job->order, job->begin);
    job->contrib.assign(size_t(n) * job->d, 0.f);
    const int ng = int(job->begin.size()) - 1;
    job->left = ng;
    {
        std::lock_guard<std::mutex> lock(eng->mu);
        for (int g = 0; g < ng; ++g) eng->tasks.push_back(MissTask{job, g});
    }
    eng->cv_work.notify_all();
}

void run_group(moe_miss_engine *eng, MissJob *job, int g, Scratch &w) {
    const moe_qmatrix *q = job->experts + size_t(job->miss[job->order[job->begin[g]]].expert) * 3;
    for (int i = job->begin[g]; i < job->begin[g + 1]; ++i) {
        const int rec = job->order[i];
        expert_record(q, job->fmt, job->d, job->f, job->x + size_t(job->miss[rec].token) * job->d, w,
                      &job->contrib[size_t(rec) * job->d]);
    }
    if (job->left.fetch_sub(1) == 1) {  // the last expert of the job: results into y, in record order
        if (job->failed) {
            finish_job(eng, MOE_ERR_HOST);
        } else {
            accumulate(job->miss, job->n, job->d, job->contrib.data(), job->y);
            finish_job(eng, MOE_OK);
        }
    }
}

void worker_loop(moe_miss_engine *eng) {
    Scratch w;
    while (true) {
        MissTask t;
        {
            std::unique_lock<std::mutex> lock(eng->mu);
            eng->cv_work.wait(lock, [&] { return eng->stop || !eng->tasks.empty(); });
            if (eng->tasks.empty()) return;  // stopping
            t = eng->tasks.front();
            eng->tasks.pop_front();
        }
        try {
            if (t.group < 0)
                start_job(eng, t.job);
            else
                run_group(eng, t.job, t.group, w);
        } catch (...) {  // host memory ran out inside a task: the job fails, y untouched
            t.job->failed = true;
            if (t.group < 0 || t.job->left.fetch_sub(1) == 1) finish_job(eng, MOE_ERR_HOST);
        }
    }
}

}  // namespace
}  // namespace moe

using namespace moe;

MOE_API moe_status moe_complete_misses_host(int fmt, int d, int f, const moe_qmatrix *experts, int E,
                                            const moe_miss *miss, int32_t n, int32_t layer, const uint16_t *x,
                                            int T, float *y, int nthreads) {
    if (E <= 0 || n < 0 || T < 0 || nthreads < 0) return MOE_ERR_INVALID_ARG;
    if (fmt != 2 && fmt != 3) return MOE_ERR_INVALID_ARG;
    if (!dims_ok(d, f)) return MOE_ERR_UNSUPPORTED;
    if (n == 0) return MOE_OK;
    if (!experts || !miss || !x || !y) return MOE_ERR_INVALID_ARG;
    const moe_status st = check_records(fmt, experts, E, miss, n, layer, T);
    if (st != MOE_OK) return st;
    try {
        return complete_misses(fmt, d, f, experts, miss, n, x, y, nthreads);
    } catch (...) {  // host memory or thread creation failed; y is unchanged
        return MOE_ERR_HOST;
    }
}

MOE_API moe_status moe_miss_engine_create(int nthreads, moe_miss_engine **engine) {
    if (!engine || nthreads < 0) return MOE_ERR_INVALID_ARG;
    *engine = nullptr;
    moe_miss_engine *eng = nullptr;
    try {
        eng = new moe_miss_engine();
        const int hw = int(std::max(1u, std::thread::hardware_concurrency()));
        const int n = nthreads > 0 ? nthreads : hw;
        for (int t = 0; t < n; ++t) eng->workers.emplace_back(worker_loop, eng);
    } catch (...) {
        if (eng) {
            {
                std::lock_guard<std::mutex> lock(eng->mu);
                eng->stop = true;
            }
            eng->cv_work.notify_all();
            for (auto &th : eng->workers) th.join();
            delete eng;
        }
        return MOE_ERR_HOST;
    }
    *engine = eng;
    return MOE_OK;
}

MOE_API moe_status moe_miss_engine_submit(moe_miss_engine *eng, int fmt, int d, int f, const moe_qmatrix *experts,
                                          int E, const moe_miss *miss, const int32_t *count, int32_t miss_cap,
                                          int32_t layer, const uint16_t *x, int T, float *y) {
    if (!eng || E <= 0 || T < 0 || miss_cap < 0) return MOE_ERR_INVALID_ARG;
    if (fmt != 2 && fmt != 3) return MOE_ERR_INVALID_ARG;
    if (!dims_ok(d, f)) return MOE_ERR_UNSUPPORTED;
    if (miss_cap == 0 || T == 0) return MOE_OK;
    if (!experts || !miss || !x || !y) return MOE_ERR_INVALID_ARG;
    try {
        auto job = std::make_unique<MissJob>();
        job->fmt = fmt;
        job->d = d;
        job->f = f;
        job->E = E;
        job->T = T;
        job->experts = experts;
        job->miss = miss;
        job->count = count;
        job->cap = miss_cap;
        job->layer = layer;
        job->x = x;
        job->y = y;
        std::lock_guard<std::mutex> lock(eng->mu);
        eng->tasks.push_back(MissTask{job.get(), -1});
        eng->jobs.push_back(std::move(job));
        ++eng->pending;
    } catch (...) {
        return MOE_ERR_HOST;
    }
    eng->cv_work.notify_one();
    return MOE_OK;
}

MOE_API moe_status moe_miss_engine_wait(moe_miss_engine *eng) {
    if (!eng) return MOE_ERR_INVALID_ARG;
    std::unique_lock<std::mutex> lock(eng->mu);
    eng->cv_done.wait(lock, [&] { return eng->pending == 0; });
    const moe_status st = eng->first_error;
    eng->first_error = MOE_OK;
    eng->jobs.clear();
    return st;
}

MOE_API void moe_miss_engine_destroy(moe_miss_engine *eng) {
    if (!eng) return;
    moe_miss_engine_wait(eng);
    {
        std::lock_guard<std::mutex> lock(eng->mu);
        eng->stop = true;
    }
    eng->cv_work.notify_all();
    for (auto &th : eng->workers) th.join();
    delete eng;
}
