// qmv_decode45.cuh -- decode units of two more GGUF formats named among the
// formats FlareLLM：纯Rust打造的浏览器端LLM推理引擎 reads (§量化技术的全面支持: the
// Q4_0 .. Q8_1 family and the K-quants):
//   Q4_0  32 weights / 18 B : d | qs[16]; byte j: weight j (low nibble) and
//                             weight j + 16 (high nibble);  w = d * (q - 8)
//   Q5_K 256 weights / 176 B: d | dmin | scales[12] (packed as Q4_K) | qh[32] |
//                             qs[128] (nibbles as Q4_K); the fifth bit of weight
//                             64c + l is bit 2c of qh[l], of weight 64c + 32 + l
//                             bit 2c + 1;  w = d * sc_j * q - dmin * m_j
// Same techniques as qmv_decode1.cuh / qmv_decodemt.cuh: exact integer -> f32
// conversion under a float exponent, packed f32x2 FMAs, scales applied once
// per group (one token) or once per weight before the token loop (several
// tokens, weight-stationary).  Slices: a Q4_0 block (32 weights, like Q8_0)
// or 64 weights of a Q5_K superblock (like Q4_K).
#pragma once

#include "qmv_decodemt.cuh"

namespace qmv {

// ---------------------------------------------------------------- Q4_0 --
// One token.  Slice = one block at shared address blk (2-byte aligned); groups
// gq = 0..3 are columns 4gq.. (low nibbles), gq = 4..7 columns 16 + 4(gq-4)..
// (high nibbles).  Returns d * sum (q - 8) x.
template <class XP>
__device__ __forceinline__ float q4_0_dot1(uint32_t blk, XP &&xp)
{
    const float d = half_bits_to_float(lds_u16(blk));
    uint32_t w[4];
    lds_words_a2<4>(blk + 2, w);
    float2 s[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 p02, p13, x02, x13;
        bytes4_to_f2(w[i] & 0x0F0F0F0Fu, 8.0f, p02, p13);          // q - 8, exact
        xp(i, x02, x13);
        s[0] = f2fma(p02, x02, s[0]);
        s[1] = f2fma(p13, x13, s[1]);
        bytes4_to_f2((w[i] >> 4) & 0x0F0F0F0Fu, 8.0f, p02, p13);
        xp(4 + i, x02, x13);
        s[2] = f2fma(p02, x02, s[2]);
        s[3] = f2fma(p13, x13, s[3]);
    }
    return d * (hsum2(s[0], s[1]) + hsum2(s[2], s[3]));
}

// Two consecutive Q4_0 blocks (36 bytes at a 4-byte-aligned shared address),
// 64 columns: block 0's quants straddle words 0..4 (two bytes in), block 1's
// scale is the high half of word 4 and its quants are words 5..8.  Groups
// gq = 0..15 are columns 4gq.. of the pair.
template <class XP>
__device__ __forceinline__ float q4_0_dot_pair(uint32_t a, XP &&xp)
{
    uint32_t w[9];
#pragma unroll
    for (int i = 0; i < 9; ++i) w[i] = lds_u32(a + 4u * (uint32_t)i);
    float r = 0.f;
#pragma unroll
    for (int b = 0; b < 2; ++b) {
        float2 s[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t q = b == 0 ? __byte_perm(w[i], w[i + 1], 0x5432u) : w[5 + i];
            float2 p02, p13, x02, x13;
            bytes4_to_f2(q & 0x0F0F0F0Fu, 8.0f, p02, p13);
            xp(8 * b + i, x02, x13);
            s[0] = f2fma(p02, x02, s[0]);
            s[1] = f2fma(p13, x13, s[1]);
            bytes4_to_f2((q >> 4) & 0x0F0F0F0Fu, 8.0f, p02, p13);
            xp(8 * b + 4 + i, x02, x13);
            s[2] = f2fma(p02, x02, s[2]);
            s[3] = f2fma(p13, x13, s[3]);
        }
        const float d = half_bits_to_float(b == 0 ? w[0] : w[4] >> 16);
        r = fmaf(d, hsum2(s[0], s[1]) + hsum2(s[2], s[3]), r);
    }
    return r;
}

// Several tokens.  blk[k] = shared address of row k's block; col0 = the block's
// first column.
template <int NTOK, int R, class XL>
__device__ __forceinline__ void q4_0_slice_mt(const uint32_t (&blk)[R], int col0, XL &&xl, float2 (&acc)[R][NTOK])
{
    float2 d[R];
#pragma unroll
    for (int k = 0; k < R; ++k) {
        const float dk = half_bits_to_float(lds_u16(blk[k]));
        d[k] = make_float2(dk, dk);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {             // word i: columns 4i.. (low) and 16 + 4i.. (high)
        float2 w[R][4];
#pragma unroll
        for (int k = 0; k < R; ++k) {
            uint32_t wd[1];
            lds_words_a2<1>(blk[k] + 2u + 4u * (uint32_t)i, wd);
            float2 l02, l13, h02, h13;
            bytes4_to_f2(wd[0] & 0x0F0F0F0Fu, 8.0f, l02, l13);
            bytes4_to_f2((wd[0] >> 4) & 0x0F0F0F0Fu, 8.0f, h02, h13);
            w[k][0] = f2mul(l02, d[k]);
            w[k][1] = f2mul(l13, d[k]);
            w[k][2] = f2mul(h02, d[k]);
            w[k][3] = f2mul(h13, d[k]);
        }
#pragma unroll
        for (int t = 0; t < NTOK; ++t) {
            const float4 a = xl(t, col0 + 4 * i);
            const float4 b = xl(t, col0 + 16 + 4 * i);
            const float2 xa02 = make_float2(a.x, a.z), xa13 = make_float2(a.y, a.w);
            const float2 xb02 = make_float2(b.x, b.z), xb13 = make_float2(b.y, b.w);
#pragma unroll
            for (int k = 0; k < R; ++k) {
                float2 s = acc[k][t];
                s = f2fma(w[k][0], xa02, s);
                s = f2fma(w[k][1], xa13, s);
                s = f2fma(w[k][2], xb02, s);
                s = f2fma(w[k][3], xb13, s);
                acc[k][t] = s;
            }
        }
    }
}

// ---------------------------------------------------------------- Q5_K --
// The five-bit quants of qs word i (bytes 4i..4i+3 of chunk c) with their
// fifth bits from qh word i: low nibbles take bit 2c, high nibbles bit 2c + 1.
__device__ __forceinline__ void q5k_quants(uint32_t qs, uint32_t qh, int c, uint32_t &lo, uint32_t &hi)
{
    lo = (qs & 0x0F0F0F0Fu) | (((qh >> (2 * c)) & 0x01010101u) << 4);
    hi = ((qs >> 4) & 0x0F0F0F0Fu) | (((qh >> (2 * c + 1)) & 0x01010101u) << 4);
}

// One token.  Slice = chunk c (64 weights) of the superblock at shared address
// sb (16-byte aligned).  Groups and the x sums as q4_k_dot1.
template <bool XSUM_INLINE, class XP>
__device__ __forceinline__ float q5_k_dot1(uint32_t sb, int c, const Q4kSel &sel, XP &&xp, float xsa, float xsb)
{
    float2 xs_a = make_float2(0.f, 0.f), xs_b = make_float2(0.f, 0.f);
    const uint4 hdr = lds_v4(sb);
    const uint4 ha = lds_v4(sb + 16u), hb = lds_v4(sb + 32u);
    const uint4 qa = lds_v4(sb + 48u + 32u * (uint32_t)c), qb = lds_v4(sb + 64u + 32u * (uint32_t)c);
    const uint32_t qh[8] = {ha.x, ha.y, ha.z, ha.w, hb.x, hb.y, hb.z, hb.w};
    const uint32_t qw[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
    float2 a0 = make_float2(0.f, 0.f), a1 = a0, b0 = a0, b1 = a0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        uint32_t lo, hi;
        q5k_quants(qw[i], qh[i], c, lo, hi);
        float2 lo02, lo13, hi02, hi13, xl02, xl13, xh02, xh13;
        bytes4_to_f2(lo, 0.0f, lo02, lo13);
        bytes4_to_f2(hi, 0.0f, hi02, hi13);
        xp(i, xl02, xl13);
        xp(8 + i, xh02, xh13);
        if (XSUM_INLINE) {
            xs_a = f2add(xs_a, f2add(xl02, xl13));
            xs_b = f2add(xs_b, f2add(xh02, xh13));
        }
        a0 = f2fma(lo02, xl02, a0); a1 = f2fma(lo13, xl13, a1);
        b0 = f2fma(hi02, xh02, b0); b1 = f2fma(hi13, xh13, b1);
    }
    const float2 sa2 = f2add(a0, a1), sb2 = f2add(b0, b1);
    const float sa = sa2.x + sa2.y, sbv = sb2.x + sb2.y;
    if (XSUM_INLINE) {
        xsa = xs_a.x + xs_a.y;
        xsb = xs_b.x + xs_b.y;
    }
    const uint32_t v = q4k_scales_mins(hdr.y, hdr.z, hdr.w, sel);   // bytes [sc0, sc1, m0, m1]
    float2 sc0_m0, sc1_m1;
    bytes4_to_f2(v, 0.0f, sc0_m0, sc1_m1);
    const float d = half_bits_to_float(hdr.x);
    const float dmin = half_bits_to_float(hdr.x >> 16);
    float r = (d * sc0_m0.x) * sa;
    r = fmaf(d * sc1_m1.x, sbv, r);
    r = fmaf(-dmin * sc0_m0.y, xsa, r);
    r = fmaf(-dmin * sc1_m1.y, xsb, r);
    return r;
}

// Several tokens.  sb[k] = shared address of row k's superblock (16-byte
// aligned), c = chunk; col0 = column 64c of the superblock.
template <int NTOK, int R, class XL>
__device__ __forceinline__ void q5_k_slice_mt(const uint32_t (&sb)[R], int c, const Q4kSel &sel, int col0, XL &&xl,
                                              float2 (&acc)[R][NTOK])
{
    float2 dscA[R], dmA[R], dscB[R], dmB[R];
#pragma unroll
    for (int k = 0; k < R; ++k) {
        const uint4 hdr = lds_v4(sb[k]);
        const uint32_t v = q4k_scales_mins(hdr.y, hdr.z, hdr.w, sel);
        float2 sc0_m0, sc1_m1;
        bytes4_to_f2(v, 0.0f, sc0_m0, sc1_m1);
        const float d = half_bits_to_float(hdr.x), dmin = half_bits_to_float(hdr.x >> 16);
        const float a = d * sc0_m0.x, b = d * sc1_m1.x;
        const float ma = -(dmin * sc0_m0.y), mb = -(dmin * sc1_m1.y);
        dscA[k] = make_float2(a, a); dmA[k] = make_float2(ma, ma);
        dscB[k] = make_float2(b, b); dmB[k] = make_float2(mb, mb);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {             // word i: low columns 4i.., high 32 + 4i..
        float2 w[R][4];
#pragma unroll
        for (int k = 0; k < R; ++k) {
            uint32_t lo, hi;
            q5k_quants(lds_u32(sb[k] + 48u + 32u * (uint32_t)c + 4u * (uint32_t)i),
                       lds_u32(sb[k] + 16u + 4u * (uint32_t)i), c, lo, hi);
            float2 lo02, lo13, hi02, hi13;
            bytes4_to_f2(lo, 0.0f, lo02, lo13);
            bytes4_to_f2(hi, 0.0f, hi02, hi13);
            w[k][0] = f2fma(lo02, dscA[k], dmA[k]);   // exact products, one rounding each
            w[k][1] = f2fma(lo13, dscA[k], dmA[k]);
            w[k][2] = f2fma(hi02, dscB[k], dmB[k]);
            w[k][3] = f2fma(hi13, dscB[k], dmB[k]);
        }
#pragma unroll
        for (int t = 0; t < NTOK; ++t) {
            const float4 a = xl(t, col0 + 4 * i);
            const float4 b = xl(t, col0 + 32 + 4 * i);
            const float2 xa02 = make_float2(a.x, a.z), xa13 = make_float2(a.y, a.w);
            const float2 xb02 = make_float2(b.x, b.z), xb13 = make_float2(b.y, b.w);
#pragma unroll
            for (int k = 0; k < R; ++k) {
                float2 s = acc[k][t];
                s = f2fma(w[k][0], xa02, s);
                s = f2fma(w[k][1], xa13, s);
                s = f2fma(w[k][2], xb02, s);
                s = f2fma(w[k][3], xb13, s);
                acc[k][t] = s;
            }
        }
    }
}

// ----------------------------------------------------- whole-block dequant --
// Exact f32 weights of one block (the dequant-only entry point).
__device__ __forceinline__ void dequant_block_q4_0(const uint8_t *blk, float *out)
{
    const float d = half_bits_to_float(blk[0] | (blk[1] << 8));
    for (int j = 0; j < 16; ++j) {
        out[j] = d * (float)((int)(blk[2 + j] & 15) - 8);
        out[j + 16] = d * (float)((int)(blk[2 + j] >> 4) - 8);
    }
}

__device__ __forceinline__ void dequant_block_q5_k(const uint8_t *blk, float *out)
{
    const float d = half_bits_to_float(blk[0] | (blk[1] << 8));
    const float dmin = half_bits_to_float(blk[2] | (blk[3] << 8));
    uint32_t s[3];
    for (int w = 0; w < 3; ++w)
        s[w] = blk[4 + 4 * w] | (blk[5 + 4 * w] << 8) | (blk[6 + 4 * w] << 16) | ((uint32_t)blk[7 + 4 * w] << 24);
    for (int j = 0; j < 8; ++j) {
        uint32_t sc, m;
        q4k_scale_min(s[0], s[1], s[2], j, sc, m);
        const float dsc = d * (float)sc;    // exact
        const float dm = dmin * (float)m;   // exact
        const int c = j >> 1, hi = j & 1;
        for (int l = 0; l < 32; ++l) {
            const uint32_t b = blk[48 + 32 * c + l];
            const uint32_t q = (hi ? (b >> 4) : (b & 15u)) | (((blk[16 + l] >> (2 * c + hi)) & 1u) << 4);
            out[32 * j + l] = __fsub_rn(__fmul_rn(dsc, (float)q), dm);   // one rounding
        }
    }
}

}  // namespace qmv
