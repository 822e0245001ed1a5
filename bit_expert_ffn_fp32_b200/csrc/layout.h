// Packed expert record: geometry and the bit placement shared by the packer
// (host and device) and the tensor-core kernels.
//
// A record holds gate [f][d], up [f][d] and down [d][f], each as a codes
// region and a scales region (256-byte aligned). Rows are cut into groups of
// 16 (the M of an m16n8k16 MMA) and K into 64-weight blocks. For lane L of a
// warp (g = L/4, t = L%4) the bits a lane needs for one MMA fragment sit in
// the same 32-bit word, so a warp fetches a (row group, k range) tile with
// coalesced 16-byte loads and unpacks each fragment register with one AND
// (plus one shift per word for the upper slots).
//
// Register slot rho (0..7) of a block = MMA i = rho/2 (k 16i..16i+15 of the
// block), half s = rho%2 (k offset 8s); inside the slot, lane t covers
// k = 16i + 8s + 2t + h for h in {0,1} (h = fp16 half of the register).
//
// Q2 (2.5 bits/weight): per (row group rg, block pair p) 512 code bytes =
//   32 lanes x 16 B; lane word w = 2*bb + r holds block 2p+bb, row g+8r;
//   slot rho's two codes sit at bits 2*rho and 2*rho+16. Scales: per (rg, p)
//   8 x 16 B; entry g = {s(g), s(g+8), m(g), m(g+8)} for block 2p, then 2p+1.
// Q3 (3.25 bits/weight): per (rg, block quad qd) 1536 code bytes =
//   3 x (32 lanes x 16 B); lane words 0..11 (word 4*sub + i at sub*512 + L*16 + 4i).
//   Unit u = 8*bq + rho (block 4qd+bq) of rows g and g+8 is placed so that both
//   rows share one power-of-two scale (see q3_place). Scales: per (rg, p) 8 x 8 B;
//   entry g = {s(g), s(g+8)} for block 2p, then 2p+1.
// A 3-bit or 2-bit field at bit offset b of a half is read as the fp16
// subnormal q * 2^(b-24); the kernels divide the activations by 2^b' (b' the
// offset after the shared shift) so that every product is q * x * 2^-24.
#pragma once

#include <stdint.h>

#ifdef __CUDACC__
#define MOE_HD __host__ __device__ __forceinline__
#else
#define MOE_HD inline
#endif

namespace moe {

struct MatGeom {
    int R, K, NG, NB;
    uint64_t codes_off, scales_off, bytes;
};

struct ExpertGeom {
    int fmt, d, f;
    MatGeom m[3];  // 0 = gate, 1 = up, 2 = down
    uint64_t bytes;
};

MOE_HD uint64_t align256(uint64_t x) { return (x + 255) & ~uint64_t(255); }

MOE_HD void mat_geom(int fmt, int R, int K, uint64_t base, MatGeom &g) {
    g.R = R;
    g.K = K;
    g.NG = R / 16;
    g.NB = K / 64;
    uint64_t code_bytes = fmt == 2 ? uint64_t(R) * K / 4 : uint64_t(R) * K * 3 / 8;
    uint64_t scale_bytes = fmt == 2 ? uint64_t(R) * K / 16 : uint64_t(R) * K / 32;
    g.codes_off = base;
    g.scales_off = base + align256(code_bytes);
    g.bytes = align256(code_bytes) + align256(scale_bytes);
}

MOE_HD ExpertGeom expert_geom(int fmt, int d, int f) {
    ExpertGeom e;
    e.fmt = fmt;
    e.d = d;
    e.f = f;
    mat_geom(fmt, f, d, 0, e.m[0]);
    mat_geom(fmt, f, d, e.m[0].bytes, e.m[1]);
    mat_geom(fmt, d, f, e.m[0].bytes + e.m[1].bytes, e.m[2]);
    e.bytes = e.m[0].bytes + e.m[1].bytes + e.m[2].bytes;
    return e;
}

// k offset inside a block of slot rho, lane t, half h.
MOE_HD int slot_k(int rho, int t, int h) { return 16 * (rho >> 1) + 8 * (rho & 1) + 2 * t + h; }

// Q2: power-of-two exponent of slot rho after extraction (bits 10..15 are
// reached through one shift by 10).
MOE_HD int q2_exp(int rho) { return rho < 5 ? 2 * rho : 2 * rho - 10; }

// Q3 placement of unit u (0..31), row r (0: g, 1: g+8), code bit j (0..2),
// half h: word index (0..11) and bit index (0..31).
MOE_HD void q3_place(int u, int r, int j, int h, int &word, int &bit) {
    if (u < 30) {
        int wp = u / 5, kind = u % 5;
        int base;
        switch (kind) {
            case 0: word = 2 * wp; base = r ? 9 : 0; break;
            case 1: word = 2 * wp; base = r ? 12 : 3; break;
            case 2: word = 2 * wp + 1; base = r ? 9 : 0; break;
            case 3: word = 2 * wp + 1; base = r ? 12 : 3; break;
            default: word = 2 * wp + r; base = 6; break;
        }
        bit = base + 16 * h + j;
    } else {
        int v = u - 30;
        word = 6 * v + 3 * r + j;
        bit = 15 + 16 * h;
    }
}

// Q3: power-of-two exponent of unit u's fp16 value.
MOE_HD int q3_exp(int u) {
    if (u >= 30) return 0;
    int kind = u % 5;
    return kind == 4 ? 6 : ((kind == 1 || kind == 3) ? 3 : 0);
}

// ---------------------------------------------------------------- canonical access
MOE_HD int canon_code(const uint8_t *codes, const uint8_t *hi, int fmt, int K, int row, int k) {
    int q = (codes[uint64_t(row) * (K / 4) + k / 4] >> (2 * (k % 4))) & 3;
    if (fmt == 3) q |= ((hi[uint64_t(row) * (K / 8) + k / 8] >> (k % 8)) & 1) << 2;
    return q;
}

MOE_HD void canon_put(uint8_t *codes, uint8_t *hi, int fmt, int K, int row, int k, int q) {
    uint8_t *c = codes + uint64_t(row) * (K / 4) + k / 4;
    *c = uint8_t((*c & ~(3 << (2 * (k % 4)))) | ((q & 3) << (2 * (k % 4))));
    if (fmt == 3) {
        uint8_t *b = hi + uint64_t(row) * (K / 8) + k / 8;
        *b = uint8_t((*b & ~(1 << (k % 8))) | (((q >> 2) & 1) << (k % 8)));
    }
}

// ---------------------------------------------------------------- one lane chunk
// Q2: the 4 words of (rg, p, lane L) from canonical codes.
MOE_HD void q2_pack_chunk(const uint8_t *codes, int K, int rg, int p, int L, uint32_t w[4]) {
    int g = L >> 2, t = L & 3;
    for (int ww = 0; ww < 4; ++ww) {
        int bb = ww >> 1, r = ww & 1;
        int row = 16 * rg + g + 8 * r;
        uint32_t v = 0;
        for (int rho = 0; rho < 8; ++rho)
            for (int h = 0; h < 2; ++h) {
                int k = 64 * (2 * p + bb) + slot_k(rho, t, h);
                v |= uint32_t(canon_code(codes, nullptr, 2, K, row, k)) << (2 * rho + 16 * h);
            }
        w[ww] = v;
    }
}

MOE_HD void q2_unpack_chunk(uint8_t *codes, int K, int rg, int p, int L, const uint32_t w[4]) {
    int g = L >> 2, t = L & 3;
    for (int ww = 0; ww < 4; ++ww) {
        int bb = ww >> 1, r = ww & 1;
        int row = 16 * rg + g + 8 * r;
        for (int rho = 0; rho < 8; ++rho)
            for (int h = 0; h < 2; ++h) {
                int k = 64 * (2 * p + bb) + slot_k(rho, t, h);
                canon_put(codes, nullptr, 2, K, row, k, int((w[ww] >> (2 * rho + 16 * h)) & 3));
            }
    }
}

// Q3: the 12 words of (rg, qd, lane L).
MOE_HD void q3_pack_chunk(const uint8_t *codes, const uint8_t *hi, int K, int rg, int qd, int L, uint32_t w[12]) {
    int g = L >> 2, t = L & 3;
    for (int i = 0; i < 12; ++i) w[i] = 0;
    for (int u = 0; u < 32; ++u)
        for (int r = 0; r < 2; ++r)
            for (int h = 0; h < 2; ++h) {
                int bq = u >> 3, rho = u & 7;
                int row = 16 * rg + g + 8 * r;
                int k = 256 * qd + 64 * bq + slot_k(rho, t, h);
                int q = canon_code(codes, hi, 3, K, row, k);
                for (int j = 0; j < 3; ++j) {
                    int word, bit;
                    q3_place(u, r, j, h, word, bit);
                    w[word] |= uint32_t((q >> j) & 1) << bit;
                }
            }
}

MOE_HD void q3_unpack_chunk(uint8_t *codes, uint8_t *hi, int K, int rg, int qd, int L, const uint32_t w[12]) {
    int g = L >> 2, t = L & 3;
    for (int u = 0; u < 32; ++u)
        for (int r = 0; r < 2; ++r)
            for (int h = 0; h < 2; ++h) {
                int bq = u >> 3, rho = u & 7;
                int row = 16 * rg + g + 8 * r;
                int k = 256 * qd + 64 * bq + slot_k(rho, t, h);
                int q = 0;
                for (int j = 0; j < 3; ++j) {
                    int word, bit;
                    q3_place(u, r, j, h, word, bit);
                    q |= int((w[word] >> bit) & 1) << j;
                }
                canon_put(codes, hi, 3, K, row, k, q);
            }
}

// Byte offsets inside a matrix region.
MOE_HD uint64_t q2_chunk_off(const MatGeom &m, int rg, int p, int L) {
    return m.codes_off + ((uint64_t(rg) * (m.NB / 2) + p) * 32 + L) * 16;
}
MOE_HD uint64_t q3_word_off(const MatGeom &m, int rg, int qd, int L, int word) {
    return m.codes_off + (uint64_t(rg) * (m.NB / 4) + qd) * 1536 + (word >> 2) * 512 + L * 16 + (word & 3) * 4;
}
// Scale entry for (rg, p, g): Q2 16 B, Q3 8 B.
MOE_HD uint64_t scale_off(const MatGeom &m, int fmt, int rg, int p, int g) {
    uint64_t e = (uint64_t(rg) * (m.NB / 2) + p) * 8 + g;
    return m.scales_off + e * (fmt == 2 ? 16 : 8);
}

}  // namespace moe
