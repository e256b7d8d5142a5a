// qmv_decode1.cuh -- one-token decode units of the quantized matvec, written
// for the fewest issued instructions per weight (the single-token matvec must
// decode ~10^13 weights/s to keep up with HBM, which leaves only a few
// instruction slots per weight).
//
// Techniques:
//   * Integer -> f32 conversion by building the float's bit pattern directly
//     (the exponent-field "magic number" method used for weight-only
//     quantized GEMMs, e.g. Kim et al. 2022, "Who Says Elephants Can't Run:
//     Bringing Large Scale MoE Models into Cloud Scale Production"): a byte u
//     placed under the exponent of 2^23 gives the float 2^23 + u, and one
//     subtraction leaves u exactly, an exact small integer.
//   * Packed f32x2 FMAs (sm_100) with several independent accumulators.
//   * The factored form per scale group: sum_i w_i x_i =
//     scale * sum_i q_i x_i (- min * sum_i x_i), so scales are applied once per
//     group, never per weight.
//
// x arrives as float2 pairs (x[c], x[c+2]) and (x[c+1], x[c+3]) for each group
// of four consecutive columns c..c+3 -- the order the conversions produce.
#pragma once

#include "qmv_device.cuh"

namespace qmv {

__device__ __forceinline__ float2 f2add(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 f2fma(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

// Four unsigned bytes of w -> (b0 - bias, b2 - bias), (b1 - bias, b3 - bias) as exact f32.
__device__ __forceinline__ void bytes4_to_f2(uint32_t w, float bias, float2 &p02, float2 &p13)
{
    const float nb = -(8388608.0f + bias);
    const float2 a = make_float2(__uint_as_float(__byte_perm(w, 0x4B000000u, 0x7650u)),
                                 __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7652u)));
    const float2 b = make_float2(__uint_as_float(__byte_perm(w, 0x4B000000u, 0x7651u)),
                                 __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7653u)));
    p02 = f2add(a, make_float2(nb, nb));
    p13 = f2add(b, make_float2(nb, nb));
}

// Eight nibbles of w as exact f32: the low nibbles (lo02, lo13) and the high
// nibbles (hi02, hi13), each pair in the order of bytes4_to_f2.
__device__ __forceinline__ void nibbles8_to_f2(uint32_t w, float2 &lo02, float2 &lo13, float2 &hi02, float2 &hi13)
{
    bytes4_to_f2(w & 0x0F0F0F0Fu, 0.0f, lo02, lo13);
    bytes4_to_f2((w >> 4) & 0x0F0F0F0Fu, 0.0f, hi02, hi13);
}

__device__ __forceinline__ float hsum2(float2 a, float2 b) { return (a.x + a.y) + (b.x + b.y); }

// ---------------------------------------------------------------- Q8_0 --
// Slice = one block (32 weights) at shared address blk (2-byte aligned).
// Groups gq = 0..7 are columns 4gq..4gq+3 of the block.  Returns d * sum q x.
template <class XP>
__device__ __forceinline__ float q8_0_dot1(uint32_t blk, XP &&xp)
{
    const float d = half_bits_to_float(lds_u16(blk));
    uint32_t w[8];
    lds_words_a2<8>(blk + 2, w);
    float2 s[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
    for (int gq = 0; gq < 8; ++gq) {
        float2 p02, p13, x02, x13;
        bytes4_to_f2(w[gq] ^ 0x80808080u, 128.0f, p02, p13);     // int8 q = byte ^ 0x80 - 128
        xp(gq, x02, x13);
        s[(gq & 1) * 2 + 0] = f2fma(p02, x02, s[(gq & 1) * 2 + 0]);
        s[(gq & 1) * 2 + 1] = f2fma(p13, x13, s[(gq & 1) * 2 + 1]);
    }
    return d * (hsum2(s[0], s[1]) + hsum2(s[2], s[3]));
}

// ---------------------------------------------------------------- Q4_K --
// The lane's per-superblock constants for chunk c (sub-blocks 2c and 2c+1):
// byte selectors that gather the sub-blocks' 6-bit scale / min fields.
struct Q4kSel {
    uint32_t sel_lo;    // c < 2: [s[j0], s[j1], s[j0+4], s[j1+4]] from (s0, s1); c >= 2: low-nibble bytes from (s2, s2)
    uint32_t sel_hi;    // c >= 2: [s[j0-4], s[j1-4], s[j0], s[j1]] from (s0, s1)
    bool upper;         // c >= 2
    uint32_t magic;     // 0x4B000000 (the bits of 2^23), held in a register
};

__device__ __forceinline__ Q4kSel q4k_sel(int c)
{
    Q4kSel s;
    const uint32_t j0 = 2u * (uint32_t)c, j1 = j0 + 1u;
    s.upper = c >= 2;
    asm volatile("mov.u32 %0, 0x4B000000;" : "=r"(s.magic));
    if (!s.upper) {
        s.sel_lo = j0 | (j1 << 4) | ((j0 + 4u) << 8) | ((j1 + 4u) << 12);
        s.sel_hi = 0;
    } else {
        // scales bytes j0+4, j1+4 live in s2 at indices j0-4, j1-4
        s.sel_lo = (j0 - 4u) | ((j1 - 4u) << 4) | ((j0 - 4u) << 8) | ((j1 - 4u) << 12);
        // s[j0-4], s[j1-4] from s0; s[j0], s[j1] from s1 (pool index 4 + j - 4 = j)
        s.sel_hi = (j0 - 4u) | ((j1 - 4u) << 4) | (j0 << 8) | (j1 << 12);
    }
    return s;
}

// [sc_j0, sc_j1, m_j0, m_j1] as bytes, from the scale words s0, s1, s2.
__device__ __forceinline__ uint32_t q4k_scales_mins(uint32_t s0, uint32_t s1, uint32_t s2, const Q4kSel &sel)
{
    const uint32_t a = __byte_perm(s0, s1, sel.sel_lo) & 0x3F3F3F3Fu;
    const uint32_t l = __byte_perm(s2, s2, sel.sel_lo);
    const uint32_t h = __byte_perm(s0, s1, sel.sel_hi);
    const uint32_t b = (l & 0x00000F0Fu) | ((l >> 4) & 0x0F0F0000u) | ((h >> 2) & 0x30303030u);
    return sel.upper ? b : a;
}

// Slice = chunk c (64 weights) of the superblock at shared address sb
// (16-byte aligned): qs bytes [32c, 32c+32); byte l's low nibble is weight
// 64c + l (sub-block 2c), its high nibble weight 64c + 32 + l (sub-block 2c+1).
// Groups gq = 0..7: low-nibble columns 64c + 4gq.., gq = 8..15: high-nibble
// columns 64c + 32 + 4(gq-8)..  xsa / xsb: sums of the slice's 32 low / high x.
template <bool XSUM_INLINE, class XP>
__device__ __forceinline__ float q4_k_dot1(uint32_t sb, int c, const Q4kSel &sel, XP &&xp, float xsa, float xsb)
{
    float2 xs_a = make_float2(0.f, 0.f), xs_b = make_float2(0.f, 0.f);
    const uint4 hdr = lds_v4(sb);
    const uint4 qa = lds_v4(sb + 16u + 32u * (uint32_t)c);
    const uint4 qb = lds_v4(sb + 32u + 32u * (uint32_t)c);
    const uint32_t qw[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
    float2 a[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
    float2 b[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
    float2 a2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
    float2 b2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float2 lo02, lo13, hi02, hi13, xl02, xl13, xh02, xh13;
        nibbles8_to_f2(qw[i], lo02, lo13, hi02, hi13);
        xp(i, xl02, xl13);
        xp(8 + i, xh02, xh13);
        if (XSUM_INLINE) {
            xs_a = f2add(xs_a, f2add(xl02, xl13));
            xs_b = f2add(xs_b, f2add(xh02, xh13));
        }
        if (i & 1) {
            a2[0] = f2fma(lo02, xl02, a2[0]); a2[1] = f2fma(lo13, xl13, a2[1]);
            b2[0] = f2fma(hi02, xh02, b2[0]); b2[1] = f2fma(hi13, xh13, b2[1]);
        } else {
            a[0] = f2fma(lo02, xl02, a[0]); a[1] = f2fma(lo13, xl13, a[1]);
            b[0] = f2fma(hi02, xh02, b[0]); b[1] = f2fma(hi13, xh13, b[1]);
        }
    }
    const float sa = hsum2(a[0], a[1]) + hsum2(a2[0], a2[1]);
    const float sbv = hsum2(b[0], b[1]) + hsum2(b2[0], b2[1]);
    if (XSUM_INLINE) {
        xsa = xs_a.x + xs_a.y;
        xsb = xs_b.x + xs_b.y;
    }
    const uint32_t v = q4k_scales_mins(hdr.y, hdr.z, hdr.w, sel);   // bytes [sc0, sc1, m0, m1]
    float2 sc0_m0, sc1_m1;
    bytes4_to_f2(v, 0.0f, sc0_m0, sc1_m1);
    const float d = half_bits_to_float(hdr.x);
    const float dmin = half_bits_to_float(hdr.x >> 16);
    // d*sc0*sa + d*sc1*sb - dmin*m0*xsa - dmin*m1*xsb
    float r = (d * sc0_m0.x) * sa;
    r = fmaf(d * sc1_m1.x, sbv, r);
    r = fmaf(-dmin * sc0_m0.y, xsa, r);
    r = fmaf(-dmin * sc1_m1.y, xsb, r);
    return r;
}

// Q4_K slice against x whose groups are pre-scaled by the powers of two that
// q4k_prescale_x applies.  Every nibble becomes a float with one bitwise op:
// a nibble at bit s of a 32-bit word, s <= 16, masked and placed under the
// exponent of 2^23 reads 2^23 + q 2^s, and one subtraction leaves q 2^s
// exactly; x carries the matching 2^-s, so each product is the same q x as
// with unscaled values (the masks replace the nibble split and the byte
// permutes of q4_k_dot1: 9 integer ops per 8 weights instead of 11).  The
// nibbles at bits 20..31 are read from v = w >> 16.
//   low nibbles (sub-block 2c):  byte 0 at bit 0, byte 1 at bit 8, byte 2 at
//     bit 16 (from w), byte 3 at bit 8 (from v)
//   high nibbles (2c + 1):      bytes 0 / 1 at bits 4 / 12 of w, bytes 2 / 3
//     at bits 4 / 12 of v
template <uint32_t MASK>
__device__ __forceinline__ float nib_f(uint32_t w, uint32_t magic)
{
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(w), "n"(MASK), "r"(magic));   // (w & MASK) | magic
    return __uint_as_float(r);
}

__device__ __forceinline__ void q4k_prescale_x(float2 (&xr)[16][2])
{
#pragma unroll
    for (int gq = 0; gq < 16; ++gq) {
        if (gq < 8) {
            xr[gq][0].y *= 0x1p-16f;
            xr[gq][1].x *= 0x1p-8f;
            xr[gq][1].y *= 0x1p-8f;
        } else {
            xr[gq][0].x *= 0x1p-4f;
            xr[gq][0].y *= 0x1p-4f;
            xr[gq][1].x *= 0x1p-12f;
            xr[gq][1].y *= 0x1p-12f;
        }
    }
}

template <class XP>
__device__ __forceinline__ float q4_k_dot1s(uint32_t sb, int c, const Q4kSel &sel, XP &&xp, float xsa, float xsb)
{
    const uint4 qa = lds_v4(sb + 16u + 32u * (uint32_t)c);
    const uint4 qb = lds_v4(sb + 32u + 32u * (uint32_t)c);
    const uint32_t qw[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
    const float2 nb = make_float2(-8388608.0f, -8388608.0f);
    const uint32_t mg = sel.magic;
    float2 a0 = make_float2(0.f, 0.f), a1 = a0, b0 = a0, b1 = a0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint32_t w = qw[i];
        const uint32_t v = w >> 16;
        const float2 lo02 = f2add(make_float2(nib_f<0x0000000Fu>(w, mg), nib_f<0x000F0000u>(w, mg)), nb);
        const float2 lo13 = f2add(make_float2(nib_f<0x00000F00u>(w, mg), nib_f<0x00000F00u>(v, mg)), nb);
        const float2 hi02 = f2add(make_float2(nib_f<0x000000F0u>(w, mg), nib_f<0x000000F0u>(v, mg)), nb);
        const float2 hi13 = f2add(make_float2(nib_f<0x0000F000u>(w, mg), nib_f<0x0000F000u>(v, mg)), nb);
        float2 xl02, xl13, xh02, xh13;
        xp(i, xl02, xl13);
        xp(8 + i, xh02, xh13);
        a0 = f2fma(lo02, xl02, a0);
        a1 = f2fma(lo13, xl13, a1);
        b0 = f2fma(hi02, xh02, b0);
        b1 = f2fma(hi13, xh13, b1);
    }
    const float2 sa2 = f2add(a0, a1), sb2 = f2add(b0, b1);
    const float sa = sa2.x + sa2.y, sbv = sb2.x + sb2.y;
    const uint4 hdr = lds_v4(sb);
    const uint32_t sv = q4k_scales_mins(hdr.y, hdr.z, hdr.w, sel);  // bytes [sc0, sc1, m0, m1]
    float2 sc0_m0, sc1_m1;
    bytes4_to_f2(sv, 0.0f, sc0_m0, sc1_m1);
    const float d = half_bits_to_float(hdr.x);
    const float dmin = half_bits_to_float(hdr.x >> 16);
    float r = (d * sc0_m0.x) * sa;
    r = fmaf(d * sc1_m1.x, sbv, r);
    r = fmaf(-dmin * sc0_m0.y, xsa, r);
    r = fmaf(-dmin * sc1_m1.y, xsb, r);
    return r;
}

// ---------------------------------------------------------------- Q6_K --
// Slice = 64 weights of the superblock at shared address sb (2-byte
// aligned): half h, l0 in {0, 16}: weights 128h + 32t + l0 + e (t = 0..3,
// e = 0..15), low 4 bits in ql[64h + l0 + e] (t = 0 low nibble, t = 2 high)
// and ql[64h + 32 + l0 + e] (t = 1 low, t = 3 high), high 2 bits at bits
// 2t..2t+1 of qh[32h + l0 + e]; scale scales[8h + 2t + l0/16].
// Groups gq = 4t + i: columns 128h + 32t + l0 + 4i...
template <class XP>
__device__ __forceinline__ float q6_k_dot1(uint32_t sb, int h, int l0, XP &&xp)
{
    uint32_t A[4], B[4], H[4], S[2];
    lds_words_a2<4>(sb + (uint32_t)(64 * h + l0), A);
    lds_words_a2<4>(sb + (uint32_t)(64 * h + 32 + l0), B);
    lds_words_a2<4>(sb + 128u + (uint32_t)(32 * h + l0), H);
    lds_words_a2<2>(sb + 192u + 8u * (uint32_t)h, S);       // scales[8h .. 8h+7]
    const float d = half_bits_to_float(lds_u16(sb + 208u));
    float2 acc[4];                                   // one packed accumulator per scale group
#pragma unroll
    for (int t = 0; t < 4; ++t) acc[t] = make_float2(0.f, 0.f);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t q[4] = {
            (A[i] & 0x0F0F0F0Fu) | ((H[i] << 4) & 0x30303030u),
            (B[i] & 0x0F0F0F0Fu) | ((H[i] << 2) & 0x30303030u),
            ((A[i] >> 4) & 0x0F0F0F0Fu) | (H[i] & 0x30303030u),
            ((B[i] >> 4) & 0x0F0F0F0Fu) | ((H[i] >> 2) & 0x30303030u)};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            float2 p02, p13, x02, x13;
            bytes4_to_f2(q[t], 32.0f, p02, p13);
            xp(4 * t + i, x02, x13);
            acc[t] = f2fma(p13, x13, f2fma(p02, x02, acc[t]));
        }
    }
    // scales for t = 0..3: bytes (l0/16) + {0, 2, 4, 6} of S
    const uint32_t o = (uint32_t)(l0 >> 4);
    const uint32_t sv = __byte_perm(S[0], S[1], o | ((o + 2u) << 4) | ((o + 4u) << 8) | ((o + 6u) << 12));
    float2 s02, s13;
    bytes4_to_f2(sv ^ 0x80808080u, 128.0f, s02, s13);        // int8 scales (t0, t2), (t1, t3)
    float r = s02.x * (acc[0].x + acc[0].y);
    r = fmaf(s13.x, acc[1].x + acc[1].y, r);
    r = fmaf(s02.y, acc[2].x + acc[2].y, r);
    r = fmaf(s13.y, acc[3].x + acc[3].y, r);
    return d * r;
}

// Column (within the chunk) of group gq of one-token slice s.
template <int FMT>
__device__ __forceinline__ int slice1_group_col(int s, int gq)
{
    if (small_block<FMT>()) {
        return 32 * s + 4 * gq;
    } else if (q4k_like<FMT>()) {
        const int sb = s >> 2, c = s & 3;
        return 256 * sb + 64 * c + (gq < 8 ? 4 * gq : 32 + 4 * (gq - 8));
    } else {
        const int sb = s >> 2, h = (s >> 1) & 1, l0 = 16 * (s & 1);
        return 256 * sb + 128 * h + 32 * (gq >> 2) + l0 + 4 * (gq & 3);
    }
}

template <int FMT> struct Slice1 {
    static constexpr int W = small_block<FMT>() ? 32 : 64;   // weights per lane slice
    static constexpr int G = W / 4;                          // groups of four columns
};

}  // namespace qmv
