// Packing canonical expert storage into the library's record (host and device).
#include <string.h>

#include "common.cuh"
#include "layout.h"

namespace moe {
namespace {

struct CanonMat {
    const uint8_t *codes;
    const uint8_t *hi;
    const uint16_t *scale;
    const uint16_t *min;
};

MOE_HD void pack_codes_one(const CanonMat &c, const MatGeom &m, int fmt, int rg, int ch, int L, uint8_t *dst) {
    if (fmt == 2) {
        uint32_t w[4];
        q2_pack_chunk(c.codes, m.K, rg, ch, L, w);
        uint8_t *o = dst + q2_chunk_off(m, rg, ch, L);
        for (int i = 0; i < 4; ++i) memcpy(o + 4 * i, &w[i], 4);
    } else {
        uint32_t w[12];
        q3_pack_chunk(c.codes, c.hi, m.K, rg, ch, L, w);
        for (int i = 0; i < 12; ++i) memcpy(dst + q3_word_off(m, rg, ch, L, i), &w[i], 4);
    }
}

MOE_HD void pack_scales_one(const CanonMat &c, const MatGeom &m, int fmt, int rg, int p, int g, uint8_t *dst) {
    uint16_t v[8];
    int nb = m.NB;
    for (int bb = 0; bb < 2; ++bb) {
        int b = 2 * p + bb;
        int r0 = 16 * rg + g, r1 = r0 + 8;
        if (fmt == 2) {
            v[4 * bb + 0] = c.scale[uint64_t(r0) * nb + b];
            v[4 * bb + 1] = c.scale[uint64_t(r1) * nb + b];
            v[4 * bb + 2] = c.min[uint64_t(r0) * nb + b];
            v[4 * bb + 3] = c.min[uint64_t(r1) * nb + b];
        } else {
            v[2 * bb + 0] = c.scale[uint64_t(r0) * nb + b];
            v[2 * bb + 1] = c.scale[uint64_t(r1) * nb + b];
        }
    }
    memcpy(dst + scale_off(m, fmt, rg, p, g), v, fmt == 2 ? 16 : 8);
}

MOE_HD void unpack_scales_one(CanonMat &c, const MatGeom &m, int fmt, int rg, int p, int g, const uint8_t *src) {
    uint16_t v[8];
    memcpy(v, src + scale_off(m, fmt, rg, p, g), fmt == 2 ? 16 : 8);
    int nb = m.NB;
    uint16_t *scale = const_cast<uint16_t *>(c.scale);
    uint16_t *mn = const_cast<uint16_t *>(c.min);
    for (int bb = 0; bb < 2; ++bb) {
        int b = 2 * p + bb;
        int r0 = 16 * rg + g, r1 = r0 + 8;
        if (fmt == 2) {
            scale[uint64_t(r0) * nb + b] = v[4 * bb + 0];
            scale[uint64_t(r1) * nb + b] = v[4 * bb + 1];
            mn[uint64_t(r0) * nb + b] = v[4 * bb + 2];
            mn[uint64_t(r1) * nb + b] = v[4 * bb + 3];
        } else {
            scale[uint64_t(r0) * nb + b] = v[2 * bb + 0];
            scale[uint64_t(r1) * nb + b] = v[2 * bb + 1];
        }
    }
}

inline int chunks_per_group(const MatGeom &m, int fmt) { return fmt == 2 ? m.NB / 2 : m.NB / 4; }

__global__ void pack_codes_kernel(CanonMat c, MatGeom m, int fmt, uint8_t *dst) {
    int nch = fmt == 2 ? m.NB / 2 : m.NB / 4;
    int64_t total = int64_t(m.NG) * nch * 32;
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < total; i += int64_t(gridDim.x) * blockDim.x) {
        int L = int(i % 32);
        int ch = int((i / 32) % nch);
        int rg = int(i / (32 * int64_t(nch)));
        pack_codes_one(c, m, fmt, rg, ch, L, dst);
    }
}

__global__ void pack_scales_kernel(CanonMat c, MatGeom m, int fmt, uint8_t *dst) {
    int np = m.NB / 2;
    int64_t total = int64_t(m.NG) * np * 8;
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < total; i += int64_t(gridDim.x) * blockDim.x) {
        int g = int(i % 8);
        int p = int((i / 8) % np);
        int rg = int(i / (8 * int64_t(np)));
        pack_scales_one(c, m, fmt, rg, p, g, dst);
    }
}

bool mats_ok(int fmt, const moe_qmatrix *a) {
    if (!a || !a->codes || !a->scale) return false;
    if (fmt == 2 && !a->min) return false;
    if (fmt == 3 && !a->hi) return false;
    return true;
}

CanonMat canon(const moe_qmatrix *a) { return CanonMat{a->codes, a->hi, a->scale, a->min}; }

moe_status check(int fmt, int d, int f, const moe_qmatrix *g, const moe_qmatrix *u, const moe_qmatrix *dn,
                 const void *dst) {
    if (fmt != 2 && fmt != 3) return MOE_ERR_UNSUPPORTED;
    if (!dims_ok(d, f)) return MOE_ERR_UNSUPPORTED;
    if (!mats_ok(fmt, g) || !mats_ok(fmt, u) || !mats_ok(fmt, dn) || !dst) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

MOE_API size_t moe_expert_bytes(int fmt, int d, int f) {
    if ((fmt != 2 && fmt != 3) || !dims_ok(d, f)) return 0;
    return size_t(expert_geom(fmt, d, f).bytes);
}

MOE_API moe_status moe_pack_expert(int fmt, int d, int f, const moe_qmatrix *gate, const moe_qmatrix *up,
                                   const moe_qmatrix *down, void *dst, moe_stream_t stream) {
    moe_status st = check(fmt, d, f, gate, up, down, dst);
    if (st != MOE_OK) return st;
    if (reinterpret_cast<uintptr_t>(dst) % 256) return MOE_ERR_INVALID_ARG;
    ExpertGeom eg = expert_geom(fmt, d, f);
    const moe_qmatrix *mats[3] = {gate, up, down};
    for (int i = 0; i < 3; ++i) {
        const MatGeom &m = eg.m[i];
        int64_t nc = int64_t(m.NG) * chunks_per_group(m, fmt) * 32;
        int64_t ns = int64_t(m.NG) * (m.NB / 2) * 8;
        pack_codes_kernel<<<int((nc + 255) / 256), 256, 0, as_cuda(stream)>>>(canon(mats[i]), m, fmt,
                                                                            static_cast<uint8_t *>(dst));
        pack_scales_kernel<<<int((ns + 255) / 256), 256, 0, as_cuda(stream)>>>(canon(mats[i]), m, fmt,
                                                                             static_cast<uint8_t *>(dst));
    }
    return launch_status();
}

MOE_API moe_status moe_pack_expert_host(int fmt, int d, int f, const moe_qmatrix *gate, const moe_qmatrix *up,
                                        const moe_qmatrix *down, void *dst_host) {
    moe_status st = check(fmt, d, f, gate, up, down, dst_host);
    if (st != MOE_OK) return st;
    ExpertGeom eg = expert_geom(fmt, d, f);
    uint8_t *dst = static_cast<uint8_t *>(dst_host);
    memset(dst, 0, eg.bytes);
    const moe_qmatrix *mats[3] = {gate, up, down};
    for (int i = 0; i < 3; ++i) {
        const MatGeom &m = eg.m[i];
        CanonMat c = canon(mats[i]);
        int nch = chunks_per_group(m, fmt);
        for (int rg = 0; rg < m.NG; ++rg)
            for (int ch = 0; ch < nch; ++ch)
                for (int L = 0; L < 32; ++L) pack_codes_one(c, m, fmt, rg, ch, L, dst);
        for (int rg = 0; rg < m.NG; ++rg)
            for (int p = 0; p < m.NB / 2; ++p)
                for (int g = 0; g < 8; ++g) pack_scales_one(c, m, fmt, rg, p, g, dst);
    }
    return MOE_OK;
}

MOE_API moe_status moe_unpack_expert_host(int fmt, int d, int f, const void *record_host, moe_qmatrix *gate,
                                          moe_qmatrix *up, moe_qmatrix *down) {
    moe_status st = check(fmt, d, f, gate, up, down, record_host);
    if (st != MOE_OK) return st;
    ExpertGeom eg = expert_geom(fmt, d, f);
    const uint8_t *src = static_cast<const uint8_t *>(record_host);
    moe_qmatrix *mats[3] = {gate, up, down};
    for (int i = 0; i < 3; ++i) {
        const MatGeom &m = eg.m[i];
        CanonMat c = canon(mats[i]);
        uint8_t *codes = const_cast<uint8_t *>(c.codes);
        uint8_t *hi = const_cast<uint8_t *>(c.hi);
        memset(codes, 0, size_t(m.R) * (m.K / 4));
        if (fmt == 3) memset(hi, 0, size_t(m.R) * (m.K / 8));
        for (int rg = 0; rg < m.NG; ++rg) {
            if (fmt == 2) {
                for (int p = 0; p < m.NB / 2; ++p)
                    for (int L = 0; L < 32; ++L) {
                        uint32_t w[4];
                        memcpy(w, src + q2_chunk_off(m, rg, p, L), 16);
                        q2_unpack_chunk(codes, m.K, rg, p, L, w);
                    }
            } else {
                for (int qd = 0; qd < m.NB / 4; ++qd)
                    for (int L = 0; L < 32; ++L) {
                        uint32_t w[12];
                        for (int j = 0; j < 12; ++j) memcpy(&w[j], src + q3_word_off(m, rg, qd, L, j), 4);
                        q3_unpack_chunk(codes, hi, m.K, rg, qd, L, w);
                    }
            }
            for (int p = 0; p < m.NB / 2; ++p)
                for (int g = 0; g < 8; ++g) unpack_scales_one(c, m, fmt, rg, p, g, src);
        }
    }
    return MOE_OK;
}
