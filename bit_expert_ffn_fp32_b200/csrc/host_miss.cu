// Host completion of the miss list.
//
// Experts that have no slot in the GPU pool are not computed on the GPU: the
// lookup step lists them as (layer, expert, token, j, gate) records, and the
// host computes them, as the engine of "5070ti16g单卡跑qwen 3.8 flash next
// 新方案最高90t/s Hermes 调用60t/s" (section "为什么从 18t/s 变成 60-90t/s") does
// with the experts that stay in system RAM. This file is that host step: for
// every record, y[token] += gate * down(silu(gate_proj x) * up_proj x) with the
// weights dequantised from the expert's packed record in a host-memory pool.
//
// Work is spread over threads one expert at a time (the expert's rows are
// dequantised once per row and applied to every token that missed it); the
// per-record results are then added into y in record order, so y does not
// depend on the thread count.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <thread>
#include <vector>

#include "common.cuh"
#include "layout.h"

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

float bf16_value(uint16_t b) {
    const uint32_t u = uint32_t(b) << 16;
    float v;
    std::memcpy(&v, &u, 4);
    return v;
}

// One expert in canonical host storage (moe_unpack_expert_host fills it).
struct HostExpert {
    int fmt = 2, d = 0, f = 0;
    std::vector<uint8_t> codes[3], hi[3];
    std::vector<uint16_t> scale[3], mn[3];
    moe_qmatrix q[3];

    void resize(int fmt_, int d_, int f_) {
        fmt = fmt_;
        d = d_;
        f = f_;
        for (int i = 0; i < 3; ++i) {
            const int R = i < 2 ? f : d, K = i < 2 ? d : f;
            codes[i].assign(size_t(R) * (K / 4), 0);
            hi[i].assign(fmt == 3 ? size_t(R) * (K / 8) : 0, 0);
            scale[i].assign(size_t(R) * (K / 64), 0);
            mn[i].assign(fmt == 2 ? size_t(R) * (K / 64) : 0, 0);
            q[i].codes = codes[i].data();
            q[i].hi = fmt == 3 ? hi[i].data() : nullptr;
            q[i].scale = scale[i].data();
            q[i].min = fmt == 2 ? mn[i].data() : nullptr;
        }
    }

    // Row r of matrix i (K weights) into w: Q2 s*q + m, Q3 s*(q-4), per 64-block.
    void row(int i, int r, float *w) const {
        const int K = i < 2 ? d : f, NB = K / 64;
        const uint8_t *c = codes[i].data() + size_t(r) * (K / 4);
        const uint8_t *h = fmt == 3 ? hi[i].data() + size_t(r) * (K / 8) : nullptr;
        for (int b = 0; b < NB; ++b) {
            const float s = half_value(scale[i][size_t(r) * NB + b]);
            const float m = fmt == 2 ? half_value(mn[i][size_t(r) * NB + b]) : 0.f;
            for (int kk = 0; kk < 64; ++kk) {
                const int k = 64 * b + kk;
                int q = (c[k >> 2] >> (2 * (k & 3))) & 3;
                if (fmt == 3) q |= ((h[k >> 3] >> (k & 7)) & 1) << 2;
                w[k] = fmt == 2 ? s * float(q) + m : s * float(q - 4);
            }
        }
    }
};

// Dot product with eight interleaved partial sums (vectorisable).
float dot(const float *a, const float *b, int n) {
    float p[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    int k = 0;
    for (; k + 8 <= n; k += 8)
        for (int j = 0; j < 8; ++j) p[j] += a[k + j] * b[k + j];
    for (; k < n; ++k) p[0] += a[k] * b[k];
    return ((p[0] + p[1]) + (p[2] + p[3])) + ((p[4] + p[5]) + (p[6] + p[7]));
}

}  // namespace
}  // namespace moe

using namespace moe;

MOE_API moe_status moe_complete_misses_host(const moe_qpool *host_pool, const int32_t *slot_of, int E,
                                            const moe_miss *miss, int32_t n, int32_t layer, const uint16_t *x,
                                            int T, float *y, int nthreads) {
    if (!host_pool || E <= 0 || n < 0 || T < 0 || nthreads < 0) return MOE_ERR_INVALID_ARG;
    if (n == 0) return MOE_OK;
    if (!slot_of || !miss || !x || !y || !host_pool->base) return MOE_ERR_INVALID_ARG;
    const int fmt = host_pool->fmt, d = host_pool->d, f = host_pool->f;
    if ((fmt != 2 && fmt != 3) || !dims_ok(d, f)) return MOE_ERR_UNSUPPORTED;
    const ExpertGeom eg = expert_geom(fmt, d, f);
    if (host_pool->num_slots <= 0 || host_pool->slot_bytes < int64_t(eg.bytes)) return MOE_ERR_INVALID_ARG;
    // every record must name this layer, a valid expert and token, and a resident host slot
    for (int32_t i = 0; i < n; ++i) {
        const moe_miss &m = miss[i];
        if (m.layer != layer || m.expert < 0 || m.expert >= E || m.token < 0 || m.token >= T)
            return MOE_ERR_INVALID_ARG;
        const int32_t s = slot_of[m.expert];
        if (s < 0 || s >= host_pool->num_slots) return MOE_ERR_INVALID_ARG;
    }
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
    std::atomic<int> failed{0};
    auto worker = [&]() {
        HostExpert ex;
        ex.resize(fmt, d, f);
        std::vector<float> w(std::max(d, f)), xf, a, u, hbuf;
        while (true) {
            const int gi = next_group.fetch_add(1);
            if (gi >= ngroups) break;
            const int g0 = group_begin[gi], g1 = group_begin[gi + 1], nt = g1 - g0;
            const int e = miss[order[g0]].expert;
            const uint8_t *rec =
                static_cast<const uint8_t *>(host_pool->base) + int64_t(slot_of[e]) * host_pool->slot_bytes;
            if (moe_unpack_expert_host(fmt, d, f, rec, &ex.q[0], &ex.q[1], &ex.q[2]) != MOE_OK) {
                failed.store(1);
                continue;
            }
            xf.assign(size_t(nt) * d, 0.f);
            for (int t = 0; t < nt; ++t)
                for (int k = 0; k < d; ++k) xf[size_t(t) * d + k] = bf16_value(x[size_t(miss[order[g0 + t]].token) * d + k]);
            a.assign(size_t(nt) * f, 0.f);
            u.assign(size_t(nt) * f, 0.f);
            for (int r = 0; r < f; ++r) {  // gate and up rows, each dequantised once for all tokens
                ex.row(0, r, w.data());
                for (int t = 0; t < nt; ++t) a[size_t(t) * f + r] = dot(w.data(), &xf[size_t(t) * d], d);
                ex.row(1, r, w.data());
                for (int t = 0; t < nt; ++t) u[size_t(t) * f + r] = dot(w.data(), &xf[size_t(t) * d], d);
            }
            hbuf.assign(size_t(nt) * f, 0.f);
            for (size_t i = 0; i < hbuf.size(); ++i) hbuf[i] = a[i] / (1.0f + std::exp(-a[i])) * u[i];
            for (int r = 0; r < d; ++r) {  // down rows
                ex.row(2, r, w.data());
                for (int t = 0; t < nt; ++t)
                    contrib[size_t(order[g0 + t]) * d + r] = dot(w.data(), &hbuf[size_t(t) * f], f);
            }
        }
    };
    const int hw = int(std::max(1u, std::thread::hardware_concurrency()));
    const int nth = std::max(1, std::min(nthreads > 0 ? nthreads : hw, ngroups));
    std::vector<std::thread> pool;
    for (int t = 1; t < nth; ++t) pool.emplace_back(worker);
    worker();
    for (auto &th : pool) th.join();
    if (failed.load()) return MOE_ERR_INVALID_ARG;
    for (int32_t i = 0; i < n; ++i) {  // record order: deterministic for any thread count
        float *yr = y + size_t(miss[i].token) * d;
        const float g = miss[i].gate;
        const float *c = &contrib[size_t(i) * d];
        for (int k = 0; k < d; ++k) yr[k] += g * c[k];
    }
    return MOE_OK;
}
