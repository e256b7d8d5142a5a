// qmv_decodemt.cuh -- multi-token (2..8 tokens) decode units.
//
// With several tokens (speculative verification -- FlareLLM：纯Rust打造的浏览器端
// LLM推理引擎, §推理层面的深度优化) each weight feeds NTOK FMAs, so the matvec
// becomes FMA- and load-bound rather than purely HBM-bound.  The units below
// therefore work "weight-stationary" on a lane's slice for all R rows of a
// warp at once: per step they decode a few weights of every row, apply the
// block scales once (the weights become exact f32 values), then stream the
// matching x values of each token once and spend them on all R rows.  Each x
// load thus feeds 2 * R packed FMAs.
//
// Slices match the one-token units (qmv_decode1.cuh): a Q8_0 block of 32
// weights, or 64 weights of a Q4_K / Q6_K superblock.  acc[k][t] is a float2
// partial sum of row k, token t.
#pragma once

#include "qmv_decode1.cuh"

namespace qmv {

// Staged x in shared memory: float4 group f of a token row lives at group
// f ^ (((f >> 3) ^ (f >> 4)) & 7), so lanes reading the same offset of
// consecutive slices fall in different banks.
__device__ __forceinline__ uint32_t xs_swizzle(uint32_t f)
{
    return f ^ (((f >> 3) ^ (f >> 4)) & 7u);
}

__device__ __forceinline__ float2 f2mul(float2 a, float2 b) { return __fmul2_rn(a, b); }

// x accessors: xl(t, col) returns x[t][col .. col+3] as a float4 (col a
// multiple of 4, relative to the current K-chunk).
//
// Q8_0: blk[k] = shared address of row k's block (2-byte aligned); col0 = the
// block's first column.
template <int NTOK, int R, class XL>
__device__ __forceinline__ void q8_0_slice_mt(const uint32_t (&blk)[R], int col0, XL &&xl,
                                              float2 (&acc)[R][NTOK])
{
    float2 d[R];
#pragma unroll
    for (int k = 0; k < R; ++k) {
        const float dk = half_bits_to_float(lds_u16(blk[k]));
        d[k] = make_float2(dk, dk);
    }
#pragma unroll
    for (int st = 0; st < 4; ++st) {           // 8 weights per step: columns 8st .. 8st+7
        float2 w[R][4];
#pragma unroll
        for (int k = 0; k < R; ++k) {
            uint32_t wd[2];
            lds_words_a2<2>(blk[k] + 2u + 8u * (uint32_t)st, wd);
            float2 p02, p13, p46, p57;
            bytes4_to_f2(wd[0] ^ 0x80808080u, 128.0f, p02, p13);
            bytes4_to_f2(wd[1] ^ 0x80808080u, 128.0f, p46, p57);
            w[k][0] = f2mul(p02, d[k]);
            w[k][1] = f2mul(p13, d[k]);
            w[k][2] = f2mul(p46, d[k]);
            w[k][3] = f2mul(p57, d[k]);
        }
#pragma unroll
        for (int t = 0; t < NTOK; ++t) {
            const float4 a = xl(t, col0 + 8 * st);
            const float4 b = xl(t, col0 + 8 * st + 4);
            const float2 x02 = make_float2(a.x, a.z), x13 = make_float2(a.y, a.w);
            const float2 x46 = make_float2(b.x, b.z), x57 = make_float2(b.y, b.w);
#pragma unroll
            for (int k = 0; k < R; ++k) {
                float2 s = acc[k][t];
                s = f2fma(w[k][0], x02, s);
                s = f2fma(w[k][1], x13, s);
                s = f2fma(w[k][2], x46, s);
                s = f2fma(w[k][3], x57, s);
                acc[k][t] = s;
            }
        }
    }
}

// Q4_K: sb[k] = shared address of row k's superblock (16-byte aligned), c =
// chunk; col0 = column 64c of the superblock.
template <int NTOK, int R, class XL>
__device__ __forceinline__ void q4_k_slice_mt(const uint32_t (&sb)[R], int c, const Q4kSel &sel,
                                              int col0, XL &&xl, float2 (&acc)[R][NTOK])
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
    for (int i = 0; i < 8; ++i) {             // qs word i: low columns 4i.., high 32 + 4i..
        float2 w[R][4];
#pragma unroll
        for (int k = 0; k < R; ++k) {
            const uint32_t wd = lds_u32(sb[k] + 16u + 32u * (uint32_t)c + 4u * (uint32_t)i);
            float2 lo02, lo13, hi02, hi13;
            nibbles8_to_f2(wd, lo02, lo13, hi02, hi13);
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

// Q6_K: sb[k] = shared address of row k's superblock (2-byte aligned); half h,
// l0 in {0, 16}; col0 = column 128h + l0 of the superblock.
template <int NTOK, int R, class XL>
__device__ __forceinline__ void q6_k_slice_mt(const uint32_t (&sb)[R], int h, int l0, int col0, XL &&xl,
                                              float2 (&acc)[R][NTOK])
{
    float2 dsc[R][4];
    const uint32_t o = (uint32_t)(l0 >> 4);
#pragma unroll
    for (int k = 0; k < R; ++k) {
        uint32_t S[2];
        lds_words_a2<2>(sb[k] + 192u + 8u * (uint32_t)h, S);
        const float d = half_bits_to_float(lds_u16(sb[k] + 208u));
        const uint32_t sv = __byte_perm(S[0], S[1], o | ((o + 2u) << 4) | ((o + 4u) << 8) | ((o + 6u) << 12));
        float2 s02, s13;
        bytes4_to_f2(sv ^ 0x80808080u, 128.0f, s02, s13);
        dsc[k][0] = make_float2(d * s02.x, d * s02.x);
        dsc[k][1] = make_float2(d * s13.x, d * s13.x);
        dsc[k][2] = make_float2(d * s02.y, d * s02.y);
        dsc[k][3] = make_float2(d * s13.y, d * s13.y);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {             // word i: columns 32t + 4i.. for t = 0..3
        float2 w[R][8];
#pragma unroll
        for (int k = 0; k < R; ++k) {
            uint32_t A[1], B[1], H[1];
            lds_words_a2<1>(sb[k] + (uint32_t)(64 * h + l0 + 4 * i), A);
            lds_words_a2<1>(sb[k] + (uint32_t)(64 * h + 32 + l0 + 4 * i), B);
            lds_words_a2<1>(sb[k] + 128u + (uint32_t)(32 * h + l0 + 4 * i), H);
            const uint32_t q[4] = {
                (A[0] & 0x0F0F0F0Fu) | ((H[0] << 4) & 0x30303030u),
                (B[0] & 0x0F0F0F0Fu) | ((H[0] << 2) & 0x30303030u),
                ((A[0] >> 4) & 0x0F0F0F0Fu) | (H[0] & 0x30303030u),
                ((B[0] >> 4) & 0x0F0F0F0Fu) | ((H[0] >> 2) & 0x30303030u)};
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                float2 p02, p13;
                bytes4_to_f2(q[t], 32.0f, p02, p13);
                w[k][2 * t] = f2mul(p02, dsc[k][t]);
                w[k][2 * t + 1] = f2mul(p13, dsc[k][t]);
            }
        }
#pragma unroll
        for (int n = 0; n < NTOK; ++n) {
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const float4 a = xl(n, col0 + 32 * t + 4 * i);
                const float2 x02 = make_float2(a.x, a.z), x13 = make_float2(a.y, a.w);
#pragma unroll
                for (int k = 0; k < R; ++k) {
                    float2 s = acc[k][n];
                    s = f2fma(w[k][2 * t], x02, s);
                    s = f2fma(w[k][2 * t + 1], x13, s);
                    acc[k][n] = s;
                }
            }
        }
    }
}

}  // namespace qmv
