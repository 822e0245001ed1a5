// Host completion of the miss list.
//
// Experts that have no slot in the GPU pool are not computed on the GPU: the
// lookup step lists them as (layer, expert, token, j, gate) records, and the
// host computes them, as the engine of "5070ti16g单卡跑qwen 3.8 flash next
// 新方案最高90t/s Hermes 调用60t/s" (section "为什么从 18t/s 变成 60-90t/s") does
// with the experts that stay in system RAM. This file is that host step: for
// every record, y[token] += gate * down(silu(gate_proj x) * up_proj x), the
// expert's weights read from their canonical storage in host memory.
//
// Dot products use lookup tables built once per input vector v: for every byte
// position i of a row's code bytes and every byte value c, tab[i][c] is the sum
// over the byte's four 2-bit codes q_j(c) of q_j(c) * v[4i+j] (and, for the Q3
// high-bit plane, the sum over the byte's eight bits). A 64-weight block of a
// row then costs 16 lookups (+ 8 for Q3) instead of 64 multiply-adds, and its
// scale and min are applied to the block's sum:
//   sum_k w_k v_k = s * sum_k q_k v_k + m * sum_k v_k        (Q2, w = s*q + m)
//                 = s * (sum_k q_k v_k - 4 * sum_k v_k)      (Q3, w = s*(q-4)).
// Work is spread over threads one expert at a time; the per-record results are
// added into y in record order, so y does not depend on the thread count.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
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

// Lookup tables of one input vector v[K] (see the top of the file).
struct InputTables {
    int K = 0;
    std::vector<float> low;   // [K/4][256]: sum_j ((c >> 2j) & 3) * v[4i+j]
    std::vector<float> high;  // [K/8][256]: sum_j ((c >> j) & 1) * v[8i+j] (Q3)
    std::vector<float> bsum;  // [K/64]: block sums of v

    void build(const float *v, int K_, bool q3) {
        K = K_;
        low.resize(size_t(K / 4) * 256);
        for (int i = 0; i < K / 4; ++i) {
            float t[4][4];
            for (int j = 0; j < 4; ++j)
                for (int q = 0; q < 4; ++q) t[j][q] = float(q) * v[4 * i + j];
            float *row = &low[size_t(i) * 256];
            for (int c = 0; c < 256; ++c) row[c] = (t[0][c & 3] + t[1][(c >> 2) & 3]) + (t[2][(c >> 4) & 3] + t[3][c >> 6]);
        }
        if (q3) {
            high.resize(size_t(K / 8) * 256);
            for (int i = 0; i < K / 8; ++i) {
                float lo16[16], hi16[16];  // nibble tables of bits 0-3 and 4-7
                for (int c = 0; c < 16; ++c) {
                    float a = 0.f, b = 0.f;
                    for (int j = 0; j < 4; ++j) {
                        if ((c >> j) & 1) {
                            a += v[8 * i + j];
                            b += v[8 * i + 4 + j];
                        }
                    }
                    lo16[c] = a;
                    hi16[c] = b;
                }
                float *row = &high[size_t(i) * 256];
                for (int c = 0; c < 256; ++c) row[c] = lo16[c & 15] + hi16[c >> 4];
            }
        }
        bsum.assign(K / 64, 0.f);
        for (int b = 0; b < K / 64; ++b) {
            float p[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            for (int k = 0; k < 64; k += 8)
                for (int j = 0; j < 8; ++j) p[j] += v[64 * b + k + j];
            bsum[b] = ((p[0] + p[1]) + (p[2] + p[3])) + ((p[4] + p[5]) + (p[6] + p[7]));
        }
    }
};

// Row r of a canonical matrix [R][K] against one input's tables.
float row_dot(const moe_qmatrix &m, int fmt, int K, int r, const InputTables &in) {
    const int NB = K / 64;
    const uint8_t *c = m.codes + size_t(r) * (K / 4);
    const uint8_t *h = fmt == 3 ? m.hi + size_t(r) * (K / 8) : nullptr;
    const uint16_t *sc = m.scale + size_t(r) * NB;
    const uint16_t *mn = fmt == 2 ? m.min + size_t(r) * NB : nullptr;
    const float *hv = half_table().data();
    float acc = 0.f;
    for (int b = 0; b < NB; ++b) {
        const float *lt = &in.low[size_t(16 * b) * 256];
        float p[4] = {0, 0, 0, 0};
        for (int i = 0; i < 16; i += 4)
            for (int j = 0; j < 4; ++j) p[j] += lt[size_t(i + j) * 256 + c[16 * b + i + j]];
        float qv = (p[0] + p[1]) + (p[2] + p[3]);
        const float s = hv[sc[b]];
        if (fmt == 2) {
            acc += s * qv + hv[mn[b]] * in.bsum[b];
        } else {
            const float *ht = &in.high[size_t(8 * b) * 256];
            float hq = 0.f;
            for (int i = 0; i < 8; ++i) hq += ht[size_t(i) * 256 + h[8 * b + i]];
            acc += s * ((qv + 4.0f * hq) - 4.0f * in.bsum[b]);
        }
    }
    return acc;
}

bool matrix_ok(const moe_qmatrix &m, int fmt) {
    return m.codes && m.scale && (fmt == 2 ? m.min != nullptr : m.hi != nullptr);
}

moe_status complete_misses(int fmt, int d, int f, const moe_qmatrix *experts, const moe_miss *miss, int32_t n,
                           const uint16_t *x, float *y, int nthreads);

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
    // every record must name this layer, a valid expert and token, and an expert whose matrices are given
    for (int32_t i = 0; i < n; ++i) {
        const moe_miss &m = miss[i];
        if (m.layer != layer || m.expert < 0 || m.expert >= E || m.token < 0 || m.token >= T)
            return MOE_ERR_INVALID_ARG;
        const moe_qmatrix *q = experts + size_t(m.expert) * 3;
        if (!matrix_ok(q[0], fmt) || !matrix_ok(q[1], fmt) || !matrix_ok(q[2], fmt)) return MOE_ERR_INVALID_ARG;
    }
    try {
        return complete_misses(fmt, d, f, experts, miss, n, x, y, nthreads);
    } catch (...) {  // host memory or thread creation failed; y is unchanged
        return MOE_ERR_HOST;
    }
}

namespace moe {
namespace {
// The validated work of moe_complete_misses_host. May throw (std::bad_alloc,
// std::system_error) before y is touched; y is written only at the end.
moe_status complete_misses(int fmt, int d, int f, const moe_qmatrix *experts, const moe_miss *miss, int32_t n,
                           const uint16_t *x, float *y, int nthreads) {
    // records grouped by expert (stable: record order kept inside a group)
    std::vector<int32_t> order(n);
    for (int32_t i = 0; i < n; ++i) order[i] = i;
    std::stable_sort(order.begin(), order.end(),
                     [&](int32_t a, int32_t b) { return miss[a].expert < miss[b].expert; });
    std::vector<int32_t> group_begin;
    for (int32_t i = 0; i < n; ++i)
        if (i == 0 || miss[order[i]].expert != miss[order[i - 1]].expert) group_begin.push_back(i);
    group_begin.push_back(n);
    const int ngroups = int(group_begin.size()) - 1;

    std::vector<float> contrib(size_t(n) * d);  // FFN output of record i (without its gate)
    std::atomic<int> next_group{0};
    std::atomic<bool> failed{false};
    auto work = [&]() {
        InputTables tab;
        std::vector<float> xf(d), a(f), u(f), h(f);
        while (true) {
            const int gi = next_group.fetch_add(1);
            if (gi >= ngroups) break;
            const moe_qmatrix *q = experts + size_t(miss[order[group_begin[gi]]].expert) * 3;
            for (int g = group_begin[gi]; g < group_begin[gi + 1]; ++g) {  // one token at a time
                const int rec = order[g];
                for (int k = 0; k < d; ++k) xf[k] = bf16_value(x[size_t(miss[rec].token) * d + k]);
                tab.build(xf.data(), d, fmt == 3);
                for (int r = 0; r < f; ++r) {
                    a[r] = row_dot(q[0], fmt, d, r, tab);
                    u[r] = row_dot(q[1], fmt, d, r, tab);
                }
                for (int r = 0; r < f; ++r) h[r] = a[r] / (1.0f + std::exp(-a[r])) * u[r];
                tab.build(h.data(), f, fmt == 3);
                float *out = &contrib[size_t(rec) * d];
                for (int r = 0; r < d; ++r) out[r] = row_dot(q[2], fmt, f, r, tab);
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
    for (int32_t i = 0; i < n; ++i) {  // record order: deterministic for any thread count
        float *yr = y + size_t(miss[i].token) * d;
        const float g = miss[i].gate;
        const float *c = &contrib[size_t(i) * d];
        for (int k = 0; k < d; ++k) yr[k] += g * c[k];
    }
    return MOE_OK;
}
}  // namespace
}  // namespace moe
