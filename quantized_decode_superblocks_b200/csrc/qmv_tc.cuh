// qmv_tc.cuh -- several-token (3..8) Q8_0, Q4_K and Q6_K matvec on the tensor cores.
//
// With n_tok tokens every weight feeds n_tok products; on the CUDA cores that
// is n_tok FMAs plus n_tok x reads per weight, which made the 8-token decode
// step several times slower than the 1-token one.  Here the weights of a
// tile of 16 rows are decoded exactly (Q8_0 quants are integers in
// [-128, 127], Q4_K quants nibbles, Q6_K quants q - 32 in [-32, 31]: all
// exact in bf16) straight into the A
// fragments of mma.m16n8k16 (bf16 in, f32 accumulate), and the tokens form
// the N = 8 columns.  x is split into two bf16 halves, hi (the float's upper
// 16 bits) and lo (the remainder, rounded): two MMAs per k-step keep every
// product within 2^-16 of f32, against a tolerance of 1e-4 of sum |w x|.
// The scales are applied in f32 in registers after each 32-column block's
// MMAs (GGUF layouts: Q8_0 w = d q with one fp16 d per 32 quants; Q4_K
// w = d sc q - dmin m per 32-column sub-block, the min term taken as
// dmin m * sum x; Q6_K w = d scale (q - 32) per 16 columns), so only
// integers and the split x go through the tensor cores.
//
// Data flow: one CTA per SM (16 warps).  The CTA's x rows sit in shared
// memory already split (token-major; 32 bytes per 8 columns, 16 of hi pairs
// and 16 of lo pairs; row pitch cols * 4 + 16 bytes, so a warp's 16-byte
// loads hit all banks once) or, when they do not fit next to the rings, are
// read through L2 and split per tile.  A unit is one tile of 16 rows x 256
// columns (4352 bytes of Q8_0, 2304 of Q4_K, 224 bytes around each row's
// Q6_K superblock in a 240-byte slot: the 60-word pitch puts the eight rows a
// quad group reads in different banks), copied by `cp.async.bulk` (one copy
// per row) into a
// warp-private ring of stages on an mbarrier, as in the warp-ring kernel.
// The CTA's row tiles go to groups of `ksplit` warps; the warps of a group
// split the K-chunks of a tile, add their partial sums in a fixed order
// through shared memory (a named barrier per group) and write y.
#pragma once

#include "qmv_kernels.cuh"

namespace qmv {

constexpr int TC_KCOLS = 256;          // columns per K-chunk (a multiple of 16 bytes in Q8_0)
constexpr int TC_ROWS = 16;            // rows per tile (MMA M)
constexpr int TC_MAX_STAGES = 6;
constexpr int TC_WARPS = 16;           // warps per CTA (one CTA per SM)
constexpr int TC_Q6K_COPY = 224;       // Q6_K: bytes copied per row (16-byte-aligned cover of a 210-byte superblock)
constexpr int TC_BAR_BYTES = 1024;
__host__ __device__ constexpr int tc_part_bytes(int nw) { return 2 * nw * 512; }   // double-buffered partial tiles (16 x 8 floats per warp)

struct TcParams {
    const uint8_t *W;
    const float *x;        // [n_tok][cols]
    float *y;              // [n_tok][rows]
    int64_t rows;
    int64_t row_bytes;
    int32_t cols;
    int32_t n_tok;         // 1..8 (missing tokens are zero columns of B)
    int32_t kc_n;          // K-chunks per row
    int32_t chunk_bytes;   // bytes of one row's K-chunk (its stride along the row)
    int32_t slot_bytes;    // bytes of one row's slot in a stage (Q6_K: a 16-byte-aligned superset of the chunk)
    int32_t ksplit;        // warps per row-tile group (divides TC_NW and kc_n)
    int32_t n_rt;          // row tiles in the matrix
    int32_t rt_q, rt_r;    // CTA c owns rt_q + (c < rt_r) consecutive row tiles
    int32_t n_stage;       // ring stages per warp
    int32_t x_pitch;       // 4-byte words per token row of shared x (cols + 4)
    int *err;
    uint32_t debug_extra_tx;   // test hook: bytes expected per tile beyond those copied (0 in use)
};

__host__ __device__ constexpr uint32_t tc_round128(uint32_t b) { return (b + 127u) & ~127u; }

// Bytes 8t .. 8t + 7 of block b's quants in one row of a stage (row at
// shared address rp, 16-byte aligned; block b at rp + 34 b, its quants two
// bytes in).  Odd blocks' quants are 4-byte aligned, even blocks' straddle.
template <int B>
__device__ __forceinline__ void tc_q8_words(uint32_t rp, int t, uint32_t &u0, uint32_t &u1)
{
    if (B & 1) {
        const uint32_t a = rp + 34u * B + 2u + 8u * (uint32_t)t;
        u0 = lds_u32(a);
        u1 = lds_u32(a + 4u);
    } else {
        const uint32_t a = rp + 34u * B + 8u * (uint32_t)t;
        const uint32_t w0 = lds_u32(a), w1 = lds_u32(a + 4u), w2 = lds_u32(a + 8u);
        u0 = __byte_perm(w0, w1, 0x5432u);
        u1 = __byte_perm(w1, w2, 0x5432u);
    }
}

// The quants of block B, rows g (q[0..7]) and g + 8 (q[8..15]), columns
// 8t .. 8t + 7, as exact floats.
template <int B>
__device__ __forceinline__ void tc_q8_frag(uint32_t ra, uint32_t rb, int t, float (&q)[16])
{
    uint32_t ua0, ua1, ub0, ub1;
    tc_q8_words<B>(ra, t, ua0, ua1);
    tc_q8_words<B>(rb, t, ub0, ub1);
    float2 p[8];             // per word: (byte 0, byte 2), (byte 1, byte 3)
    bytes4_to_f2(ua0 ^ 0x80808080u, 128.0f, p[0], p[1]);
    bytes4_to_f2(ua1 ^ 0x80808080u, 128.0f, p[2], p[3]);
    bytes4_to_f2(ub0 ^ 0x80808080u, 128.0f, p[4], p[5]);
    bytes4_to_f2(ub1 ^ 0x80808080u, 128.0f, p[6], p[7]);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        q[8 * h + 0] = p[4 * h + 0].x; q[8 * h + 1] = p[4 * h + 1].x;   // columns 0, 1
        q[8 * h + 2] = p[4 * h + 0].y; q[8 * h + 3] = p[4 * h + 1].y;   // 2, 3
        q[8 * h + 4] = p[4 * h + 2].x; q[8 * h + 5] = p[4 * h + 3].x;   // 4, 5
        q[8 * h + 6] = p[4 * h + 2].y; q[8 * h + 7] = p[4 * h + 3].y;   // 6, 7
    }
}

// d[0..3] += A (16x16, bf16) * B (16x8, bf16), f32 accumulation.  Fragments
// (PTX ISA, m16n8k16; each register holds two bf16, the lower column / row
// in the low half): a0 (g; 2t, 2t+1), a1 (g + 8; 2t, 2t+1), a2 (g; 2t+8,
// 2t+9), a3 (g + 8; 2t+8, 2t+9); b0 (k = 2t, 2t+1; n = g), b1 (k = 2t+8,
// 2t+9; n = g); d as for m16n8k8.
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1)
{
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// bf16x2 {lo, hi} rounded to nearest from two floats.
__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// Columns c .. c + 7 of one x row as bf16 pairs: hi = the upper 16 bits of
// each float (exact truncation), lo = bf16 of the remainder x - hi (exact in
// f32), so |x - hi - lo| <= 2^-16 |x| and every product q (hi + lo) is
// within 2^-16 of q x.  Pair i holds columns c + 2i, c + 2i + 1.
__device__ __forceinline__ void tc_split_x8(float4 xa, float4 xb, uint4 &bh, uint4 &bl)
{
    const float xv[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
    uint32_t h[4], l[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t u0 = __float_as_uint(xv[2 * i]), u1 = __float_as_uint(xv[2 * i + 1]);
        h[i] = __byte_perm(u0, u1, 0x7632u);
        const float2 r = f2fma(make_float2(__uint_as_float(u0 & 0xFFFF0000u), __uint_as_float(u1 & 0xFFFF0000u)),
                               make_float2(-1.0f, -1.0f), make_float2(xv[2 * i], xv[2 * i + 1]));
        l[i] = bf16x2_rn(r.x, r.y);
    }
    bh = make_uint4(h[0], h[1], h[2], h[3]);
    bl = make_uint4(l[0], l[1], l[2], l[3]);
}

// B fragments of block b for thread t: x[token g][32b + 8t .. + 7] as hi /
// lo bf16 pairs.  XS: already split in shared memory (xrow: the token's row
// there, 32 bytes per 8 columns: 16 of hi pairs, 16 of lo pairs); else
// read through L2 (xg) and split here.
template <bool XS>
__device__ __forceinline__ void tc_x_frag(uint32_t xrow, const float *xg, int b, int t, bool have_x, uint4 &bh,
                                          uint4 &bl)
{
    bh = make_uint4(0u, 0u, 0u, 0u);
    bl = bh;
    if (!have_x) return;
    if (XS) {
        const uint32_t a = xrow + 32u * (uint32_t)(4 * b + t);
        bh = lds_v4(a);
        bl = lds_v4(a + 16u);
    } else {
        const float4 xa = __ldg(reinterpret_cast<const float4 *>(xg + 32 * b + 8 * t));
        const float4 xb = __ldg(reinterpret_cast<const float4 *>(xg + 32 * b + 8 * t + 4));
        tc_split_x8(xa, xb, bh, bl);
    }
}

// Two blocks on bf16 MMAs: the quants (|q| <= 128, exact in bf16) packed in
// column pairs; k-step s (0, 1) of block b gives thread t the columns
// 32b + 8t + 4s, +1 (k = 2t, 2t+1) and +2, +3 (k = 2t+8, 2t+9).
template <int B0, bool XS>
__device__ __forceinline__ void tc_q8_pair_bf16(uint32_t ra, uint32_t rb, uint32_t xrow, const float *xg, bool have_x,
                                                int t, float (&acc)[4])
{
    uint4 x0h, x0l, x1h, x1l;
    tc_x_frag<XS>(xrow, xg, B0, t, have_x, x0h, x0l);
    tc_x_frag<XS>(xrow, xg, B0 + 1, t, have_x, x1h, x1l);
    const uint32_t h0[4] = {x0h.x, x0h.y, x0h.z, x0h.w}, l0[4] = {x0l.x, x0l.y, x0l.z, x0l.w};
    const uint32_t h1[4] = {x1h.x, x1h.y, x1h.z, x1h.w}, l1[4] = {x1l.x, x1l.y, x1l.z, x1l.w};
    float q0[16], q1[16];
    tc_q8_frag<B0>(ra, rb, t, q0);
    tc_q8_frag<B0 + 1>(ra, rb, t, q1);
    uint32_t p0[8], p1[8];       // [row half h][pair i]: columns 2i, 2i + 1
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        p0[i] = bf16x2_rn(q0[2 * i], q0[2 * i + 1]);
        p1[i] = bf16x2_rn(q1[2 * i], q1[2 * i + 1]);
    }
    float c0h[4] = {0.f, 0.f, 0.f, 0.f}, c0l[4] = {0.f, 0.f, 0.f, 0.f};
    float c1h[4] = {0.f, 0.f, 0.f, 0.f}, c1l[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int s = 0; s < 2; ++s) {
        // a0: row g pair 2s; a2: row g pair 2s + 1; a1 / a3: row g + 8
        mma_bf16(c0h, p0[2 * s], p0[4 + 2 * s], p0[2 * s + 1], p0[4 + 2 * s + 1], h0[2 * s], h0[2 * s + 1]);
        mma_bf16(c1h, p1[2 * s], p1[4 + 2 * s], p1[2 * s + 1], p1[4 + 2 * s + 1], h1[2 * s], h1[2 * s + 1]);
        mma_bf16(c0l, p0[2 * s], p0[4 + 2 * s], p0[2 * s + 1], p0[4 + 2 * s + 1], l0[2 * s], l0[2 * s + 1]);
        mma_bf16(c1l, p1[2 * s], p1[4 + 2 * s], p1[2 * s + 1], p1[4 + 2 * s + 1], l1[2 * s], l1[2 * s + 1]);
    }
    const float da0 = half_bits_to_float(lds_u16(ra + 34u * B0)), db0 = half_bits_to_float(lds_u16(rb + 34u * B0));
    const float da1 = half_bits_to_float(lds_u16(ra + 34u * (B0 + 1))), db1 = half_bits_to_float(lds_u16(rb + 34u * (B0 + 1)));
    acc[0] = fmaf(da0, c0h[0] + c0l[0], acc[0]);
    acc[1] = fmaf(da0, c0h[1] + c0l[1], acc[1]);
    acc[2] = fmaf(db0, c0h[2] + c0l[2], acc[2]);
    acc[3] = fmaf(db0, c0h[3] + c0l[3], acc[3]);
    acc[0] = fmaf(da1, c1h[0] + c1l[0], acc[0]);
    acc[1] = fmaf(da1, c1h[1] + c1l[1], acc[1]);
    acc[2] = fmaf(db1, c1h[2] + c1l[2], acc[2]);
    acc[3] = fmaf(db1, c1h[3] + c1l[3], acc[3]);
}

// One 16 x 256 Q8_0 tile against the 8 token columns: acc (rows g, g + 8;
// tokens 2t, 2t + 1) += sum over the 8 blocks of d_row * (q . x).
template <bool XS>
__device__ __forceinline__ void tc_q8_tile(uint32_t st, int chunk_bytes, uint32_t xrow, const float *xg, bool have_x,
                                           int g, int t, float (&acc)[4])
{
    const uint32_t ra = st + (uint32_t)(g * chunk_bytes);
    const uint32_t rb = ra + 8u * (uint32_t)chunk_bytes;
    tc_q8_pair_bf16<0, XS>(ra, rb, xrow, xg, have_x, t, acc);
    tc_q8_pair_bf16<2, XS>(ra, rb, xrow, xg, have_x, t, acc);
    tc_q8_pair_bf16<4, XS>(ra, rb, xrow, xg, have_x, t, acc);
    tc_q8_pair_bf16<6, XS>(ra, rb, xrow, xg, have_x, t, acc);
}

// ------------------------------------------------------------------ Q4_K --
// Four quants (nibbles 0..15, one per byte of nb) of columns c .. c + 3 as
// two exact bf16 pairs: each byte under the exponent of 128 (bf16 0x43qq =
// 128 + q), then one exact bf16x2 FMA q' * 1 - 128.
__device__ __forceinline__ void tc_nib_pairs(uint32_t nb, uint32_t &p01, uint32_t &p23)
{
    const uint32_t v01 = __byte_perm(nb, 0x43434343u, 0x5140u);
    const uint32_t v23 = __byte_perm(nb, 0x43434343u, 0x7362u);
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(p01) : "r"(v01), "r"(0x3F803F80u), "r"(0xC300C300u));
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(p23) : "r"(v23), "r"(0x3F803F80u), "r"(0xC300C300u));
}

// Sub-blocks 2C (low nibbles of qs[32C .. 32C + 31]) and 2C + 1 (their high
// nibbles) of one Q4_K superblock per row (GGUF layout: d, dmin, 12 bytes of
// packed 6-bit scales / mins, 128 bytes of quants; w = d sc q - dmin m):
// sum_i w_i x_i = d sc (q . x) - dmin m (sum x), with q . x from the tensor
// cores and sum x per 32 columns and token from the table at sxc.  Thread t
// takes columns 8t .. 8t + 7 of each sub-block, as for Q8_0.
template <int C, bool XS>
__device__ __forceinline__ void tc_q4k_pair(uint32_t ra, uint32_t rb, const uint4 &ha, const uint4 &hb, float da,
                                            float dma, float db, float dmb, uint32_t xrow, const float *xg,
                                            bool have_x, int t, uint32_t sxc, float (&acc)[4])
{
    uint4 x0h, x0l, x1h, x1l;
    tc_x_frag<XS>(xrow, xg, 2 * C, t, have_x, x0h, x0l);
    tc_x_frag<XS>(xrow, xg, 2 * C + 1, t, have_x, x1h, x1l);
    const uint32_t h0[4] = {x0h.x, x0h.y, x0h.z, x0h.w}, l0[4] = {x0l.x, x0l.y, x0l.z, x0l.w};
    const uint32_t h1[4] = {x1h.x, x1h.y, x1h.z, x1h.w}, l1[4] = {x1l.x, x1l.y, x1l.z, x1l.w};
    const uint32_t off = 16u + 32u * C + 8u * (uint32_t)t;
    const uint32_t wa0 = lds_u32(ra + off), wa1 = lds_u32(ra + off + 4u);
    const uint32_t wb0 = lds_u32(rb + off), wb1 = lds_u32(rb + off + 4u);
    uint32_t p0[8], p1[8];       // [row half][pair]: columns 2i, 2i + 1 (low nibbles: p0, high: p1)
    tc_nib_pairs(wa0 & 0x0F0F0F0Fu, p0[0], p0[1]);
    tc_nib_pairs(wa1 & 0x0F0F0F0Fu, p0[2], p0[3]);
    tc_nib_pairs(wb0 & 0x0F0F0F0Fu, p0[4], p0[5]);
    tc_nib_pairs(wb1 & 0x0F0F0F0Fu, p0[6], p0[7]);
    tc_nib_pairs((wa0 >> 4) & 0x0F0F0F0Fu, p1[0], p1[1]);
    tc_nib_pairs((wa1 >> 4) & 0x0F0F0F0Fu, p1[2], p1[3]);
    tc_nib_pairs((wb0 >> 4) & 0x0F0F0F0Fu, p1[4], p1[5]);
    tc_nib_pairs((wb1 >> 4) & 0x0F0F0F0Fu, p1[6], p1[7]);
    float c0h[4] = {0.f, 0.f, 0.f, 0.f}, c0l[4] = {0.f, 0.f, 0.f, 0.f};
    float c1h[4] = {0.f, 0.f, 0.f, 0.f}, c1l[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int s = 0; s < 2; ++s) {
        mma_bf16(c0h, p0[2 * s], p0[4 + 2 * s], p0[2 * s + 1], p0[4 + 2 * s + 1], h0[2 * s], h0[2 * s + 1]);
        mma_bf16(c1h, p1[2 * s], p1[4 + 2 * s], p1[2 * s + 1], p1[4 + 2 * s + 1], h1[2 * s], h1[2 * s + 1]);
        mma_bf16(c0l, p0[2 * s], p0[4 + 2 * s], p0[2 * s + 1], p0[4 + 2 * s + 1], l0[2 * s], l0[2 * s + 1]);
        mma_bf16(c1l, p1[2 * s], p1[4 + 2 * s], p1[2 * s + 1], p1[4 + 2 * s + 1], l1[2 * s], l1[2 * s + 1]);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int j = 2 * C + h;
        uint32_t sca, ma, scb, mb;
        q4k_scale_min(ha.y, ha.z, ha.w, j, sca, ma);
        q4k_scale_min(hb.y, hb.z, hb.w, j, scb, mb);
        const float2 sx = lds_f2(sxc + 4u * (uint32_t)(8 * j + 2 * t));   // sum x of this sub-block, tokens 2t, 2t + 1
        const float *ch = h ? c1h : c0h, *cl = h ? c1l : c0l;
        const float aa = da * (float)sca, ba = dma * (float)ma, ab = db * (float)scb, bb = dmb * (float)mb;
        acc[0] = fmaf(aa, ch[0] + cl[0], fmaf(-ba, sx.x, acc[0]));
        acc[1] = fmaf(aa, ch[1] + cl[1], fmaf(-ba, sx.y, acc[1]));
        acc[2] = fmaf(ab, ch[2] + cl[2], fmaf(-bb, sx.x, acc[2]));
        acc[3] = fmaf(ab, ch[3] + cl[3], fmaf(-bb, sx.y, acc[3]));
    }
}

// One 16-row tile of one Q4_K superblock (256 columns) against the 8 token
// columns; sxc: the sum-x table of this K-chunk ([32-column block][8 tokens]).
template <bool XS>
__device__ __forceinline__ void tc_q4k_tile(uint32_t st, int chunk_bytes, uint32_t xrow, const float *xg, bool have_x,
                                            int g, int t, uint32_t sxc, float (&acc)[4])
{
    const uint32_t ra = st + (uint32_t)(g * chunk_bytes);
    const uint32_t rb = ra + 8u * (uint32_t)chunk_bytes;
    const uint4 ha = lds_v4(ra), hb = lds_v4(rb);
    const float da = half_bits_to_float(ha.x), dma = half_bits_to_float(ha.x >> 16);
    const float db = half_bits_to_float(hb.x), dmb = half_bits_to_float(hb.x >> 16);
    tc_q4k_pair<0, XS>(ra, rb, ha, hb, da, dma, db, dmb, xrow, xg, have_x, t, sxc, acc);
    tc_q4k_pair<1, XS>(ra, rb, ha, hb, da, dma, db, dmb, xrow, xg, have_x, t, sxc, acc);
    tc_q4k_pair<2, XS>(ra, rb, ha, hb, da, dma, db, dmb, xrow, xg, have_x, t, sxc, acc);
    tc_q4k_pair<3, XS>(ra, rb, ha, hb, da, dma, db, dmb, xrow, xg, have_x, t, sxc, acc);
}

// ------------------------------------------------------------------ Q6_K --
// Four bytes at a 2-byte-aligned shared address.
__device__ __forceinline__ uint32_t tc_lds_u32_a2(uint32_t a)
{
    const uint32_t a4 = a & ~3u;
    return __byte_perm(lds_u32(a4), lds_u32(a4 + 4u), (a & 2u) ? 0x5432u : 0x3210u);
}

__device__ __forceinline__ int tc_lds_s8(uint32_t a)
{
    int v;
    asm volatile("ld.shared.s8 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}

// Four 6-bit quants u (one per byte, 0..63) as two exact bf16 pairs of
// q = u - 32: each byte under the exponent of 128, then an exact bf16x2 FMA
// subtracts 160.
__device__ __forceinline__ void tc_q6_pairs(uint32_t u, uint32_t &p01, uint32_t &p23)
{
    const uint32_t v01 = __byte_perm(u, 0x43434343u, 0x5140u);
    const uint32_t v23 = __byte_perm(u, 0x43434343u, 0x7362u);
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(p01) : "r"(v01), "r"(0x3F803F80u), "r"(0xC320C320u));
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(p23) : "r"(v23), "r"(0x3F803F80u), "r"(0xC320C320u));
}

// One 16-row tile of one Q6_K superblock (GGUF layout: ql[128], qh[64],
// int8 scales[16], fp16 d; weight i of the superblock: half h = i / 128,
// quarter t = (i / 32) % 4, l = i % 32; low 4 bits from ql[64h + 32(t & 1) +
// l] (high nibble when t >= 2), high 2 bits from qh[32h + l] >> 2t;
// w = d * scales[i / 16] * (q - 32)).  One k-step per 16-column scale group:
// thread t takes its columns 4t .. 4t + 3 (k = 2t, 2t + 1 and 2t + 8,
// 2t + 9).  The superblock starts `sofs` bytes into each row's slot.
__device__ __forceinline__ void tc_q6k_tile(uint32_t st, int slot_bytes, int sofs, uint32_t xrow, bool have_x, int g,
                                            int t, float (&acc)[4])
{
    const uint32_t ra = st + (uint32_t)(g * slot_bytes + sofs);
    const uint32_t rb = ra + 8u * (uint32_t)slot_bytes;
    const float da = half_bits_to_float(lds_u16(ra + 208u)), db = half_bits_to_float(lds_u16(rb + 208u));
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        const int h = j >> 3, q4 = (j >> 1) & 3;
        const uint32_t lo_off = (uint32_t)(64 * h + 32 * (q4 & 1) + 16 * (j & 1) + 4 * t);
        const uint32_t hi_off = (uint32_t)(128 + 32 * h + 16 * (j & 1) + 4 * t);
        const int nsh = q4 >= 2 ? 4 : 0;
        const uint32_t ua = ((tc_lds_u32_a2(ra + lo_off) >> nsh) & 0x0F0F0F0Fu) |
                            (((tc_lds_u32_a2(ra + hi_off) >> (2 * q4)) & 0x03030303u) << 4);
        const uint32_t ub = ((tc_lds_u32_a2(rb + lo_off) >> nsh) & 0x0F0F0F0Fu) |
                            (((tc_lds_u32_a2(rb + hi_off) >> (2 * q4)) & 0x03030303u) << 4);
        uint32_t a01, a23, b01, b23;
        tc_q6_pairs(ua, a01, a23);
        tc_q6_pairs(ub, b01, b23);
        // x: columns 16j + 4t .. + 3 = pairs 2(t & 1), 2(t & 1) + 1 of 8-column group 2j + t / 2
        uint32_t xh0 = 0u, xh1 = 0u, xl0 = 0u, xl1 = 0u;
        if (have_x) {
            const uint32_t xa = xrow + 32u * (uint32_t)(2 * j + (t >> 1)) + 8u * (uint32_t)(t & 1);
            const uint2 vh = lds_v2(xa), vl = lds_v2(xa + 16u);
            xh0 = vh.x; xh1 = vh.y; xl0 = vl.x; xl1 = vl.y;
        }
        float ch[4] = {0.f, 0.f, 0.f, 0.f}, cl[4] = {0.f, 0.f, 0.f, 0.f};
        mma_bf16(ch, a01, b01, a23, b23, xh0, xh1);
        mma_bf16(cl, a01, b01, a23, b23, xl0, xl1);
        const float sa = da * (float)tc_lds_s8(ra + 192u + (uint32_t)j);
        const float sb = db * (float)tc_lds_s8(rb + 192u + (uint32_t)j);
        acc[0] = fmaf(sa, ch[0] + cl[0], acc[0]);
        acc[1] = fmaf(sa, ch[1] + cl[1], acc[1]);
        acc[2] = fmaf(sb, ch[2] + cl[2], acc[2]);
        acc[3] = fmaf(sb, ch[3] + cl[3], acc[3]);
    }
}

template <int FMT, int NWARP, bool XS>
__global__ void __launch_bounds__(NWARP * 32, 1) qmv_tc_kernel(const TcParams p)
{
    constexpr int TC_NW = NWARP;
    constexpr int TC_NT = NWARP * 32;
    constexpr int TC_PART_BYTES = tc_part_bytes(NWARP);
    static_assert(FMT == FMT_Q8_0 || FMT == FMT_Q4_K || (FMT == FMT_Q6_K && XS), "tensor-core path: Q8_0, Q4_K, Q6_K");
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = (int)threadIdx.x >> 5, lane = (int)threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const uint32_t sraw = smem_addr(smem);
    const uint32_t sbase = (sraw + 127u) & ~127u;          // the launch adds 128 spare bytes
    const int S = p.n_stage;
    const uint32_t bar0 = sbase + 8u * (uint32_t)(warp * TC_MAX_STAGES);
    const uint32_t xs = sbase + (uint32_t)TC_BAR_BYTES;
    const uint32_t x_bytes = XS ? tc_round128((uint32_t)(p.n_tok * p.x_pitch * 4)) : 0u;
    const uint32_t part = xs + x_bytes;
    const uint32_t tile_bytes = (uint32_t)(TC_ROWS * p.slot_bytes);
    const uint32_t sx = part + (uint32_t)TC_PART_BYTES;       // Q4_K: sum x per 32 columns, [block][8 tokens]
    const uint32_t sx_bytes = FMT == FMT_Q4_K ? tc_round128((uint32_t)p.cols) : 0u;
    const uint32_t stage0 = sx + sx_bytes + (uint32_t)(warp * S) * tile_bytes;

    // this CTA's row tiles, this warp's group and K-chunks
    const int c = (int)blockIdx.x;
    const int rt_a = c * p.rt_q + min(c, p.rt_r);
    const int n_local = p.rt_q + (c < p.rt_r ? 1 : 0);
    const int ks = p.ksplit;
    const int n_grp = TC_NW / ks;
    const int grp = warp / ks, kg = warp - grp * ks;
    const int kpw = p.kc_n / ks;                            // K-chunks per warp per tile
    const int n_rl = n_local > grp ? (n_local - grp + n_grp - 1) / n_grp : 0;   // tiles grp, grp + n_grp, ...
    const int n_units = n_rl * kpw;

    if (lane == 0) {
        for (int s = 0; s < S; ++s) mbar_init(bar0 + 8u * (uint32_t)s, 1);
        fence_mbar_init();
    }
    __syncthreads();
    pdl_launch_dependents();

    // unit j of this warp: local tile grp + (j / kpw) * n_grp, K-chunk kg * kpw + j % kpw
    auto issue = [&](int j) {
        const int rl = grp + (j / kpw) * n_grp;
        const int kc = kg * kpw + (j % kpw);
        const int64_t r0 = (int64_t)(rt_a + rl) * TC_ROWS;
        const int valid = (int)min((int64_t)TC_ROWS, p.rows - r0);
        const int sl = j % S;
        const uint32_t bar = bar0 + 8u * (uint32_t)sl;
        // Q6_K chunks (210 bytes) start on 2-byte boundaries: copy the 16-byte-aligned
        // slot around each, cut at the end of the matrix (which is 16-byte aligned)
        int64_t off = (r0 + lane) * p.row_bytes + (int64_t)kc * p.chunk_bytes;
        uint32_t size = (uint32_t)p.chunk_bytes;
        if (FMT == FMT_Q6_K) {
            off &= ~(int64_t)15;
            size = (uint32_t)min((int64_t)TC_Q6K_COPY, p.rows * p.row_bytes - off);
        }
        if (lane >= valid) size = 0u;
        const uint32_t total = __reduce_add_sync(0xffffffffu, size);
        if (lane == 0) mbar_arrive_expect_tx(bar, total + p.debug_extra_tx);
        __syncwarp();
        if (lane < valid)
            bulk_g2s(stage0 + (uint32_t)sl * tile_bytes + (uint32_t)(lane * p.slot_bytes), p.W + off, size, bar);
    };
    int issued = 0;
    for (; issued < S && issued < n_units; ++issued) issue(issued);   // weights: no dependence on earlier kernels

    pdl_wait();                                         // x is the previous kernel's output
    if (XS) {           // split once per CTA: 32 bytes per 8 columns, hi pairs then lo pairs
        const int c8 = p.cols >> 3;
        for (int i = (int)threadIdx.x; i < p.n_tok * c8; i += TC_NT) {
            const int tok = i / c8, j = i - tok * c8;
            const float4 *src = reinterpret_cast<const float4 *>(p.x + (int64_t)tok * p.cols) + 2 * j;
            uint4 h, l;
            tc_split_x8(__ldg(src), __ldg(src + 1), h, l);
            const uint32_t a = xs + 4u * (uint32_t)(tok * p.x_pitch) + 32u * (uint32_t)j;
            sts_v4(a, h);
            sts_v4(a + 16u, l);
        }
    }
    if (FMT == FMT_Q4_K) {   // sum x of every 32-column block and token (zero for the missing tokens)
        for (int i = (int)threadIdx.x; i < (p.cols >> 5) * 8; i += TC_NT) {
            const int blk = i >> 3, tok = i & 7;
            float sum = 0.f;
            if (tok < p.n_tok) {
                const float4 *src = reinterpret_cast<const float4 *>(p.x + (int64_t)tok * p.cols + 32 * blk);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const float4 v = __ldg(src + k);
                    sum += (v.x + v.y) + (v.z + v.w);
                }
            }
            sts_f32(sx + 4u * (uint32_t)i, sum);
        }
    }
    __syncthreads();

    const bool have_x = g < p.n_tok;
    const uint32_t xrow0 = xs + 4u * (uint32_t)(g * p.x_pitch);
    const float *xg0 = p.x + (int64_t)(have_x ? g : 0) * p.cols;
    bool dead = false;
    int consumed = 0;
    for (int it = 0; it < n_rl; ++it) {
        const int rl = grp + it * n_grp;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        for (int k = 0; k < kpw; ++k) {
            const int j = it * kpw + k;
            if (!dead) {
                const int sl = j % S;
                bool ok = mbar_wait_bounded(bar0 + 8u * (uint32_t)sl, (uint32_t)((j / S) & 1));
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) {
                    dead = true;
                    if (lane == 0) atomicOr(p.err, DEVERR_TIMEOUT);
                } else {
                    const int kc = kg * kpw + k;
                    if (FMT == FMT_Q8_0)
                        tc_q8_tile<XS>(stage0 + (uint32_t)sl * tile_bytes, p.chunk_bytes,
                                       xrow0 + 4u * (uint32_t)(kc * TC_KCOLS), xg0 + kc * TC_KCOLS, have_x, g, t, acc);
                    else if (FMT == FMT_Q6_K)
                        tc_q6k_tile(stage0 + (uint32_t)sl * tile_bytes, p.slot_bytes, (2 * kc) & 15,
                                    xrow0 + 4u * (uint32_t)(kc * TC_KCOLS), have_x, g, t, acc);
                    else
                        tc_q4k_tile<XS>(stage0 + (uint32_t)sl * tile_bytes, p.chunk_bytes,
                                        xrow0 + 4u * (uint32_t)(kc * TC_KCOLS), xg0 + kc * TC_KCOLS, have_x, g, t,
                                        sx + 4u * (uint32_t)(kc * (TC_KCOLS / 32) * 8), acc);
                    consumed = j + 1;
                    __syncwarp();
                    if (issued < n_units) { issue(issued); ++issued; }
                }
            }
        }
        const int64_t r0 = (int64_t)(rt_a + rl) * TC_ROWS;
        if (ks == 1) {
            const int64_t ra = r0 + g, rb = r0 + g + 8;
            const int t0 = 2 * t, t1 = 2 * t + 1;
            if (t0 < p.n_tok) {
                if (ra < p.rows) p.y[(int64_t)t0 * p.rows + ra] = acc[0];
                if (rb < p.rows) p.y[(int64_t)t0 * p.rows + rb] = acc[2];
            }
            if (t1 < p.n_tok) {
                if (ra < p.rows) p.y[(int64_t)t1 * p.rows + ra] = acc[1];
                if (rb < p.rows) p.y[(int64_t)t1 * p.rows + rb] = acc[3];
            }
        } else {
            // partial tile [token 8][row 16] of warp kg in buffer it & 1 of the group
            const uint32_t pb = part + (uint32_t)((((it & 1) * TC_NW) + grp * ks) * 512);
            const uint32_t mine = pb + (uint32_t)(kg * 512);
            sts_f32(mine + 4u * (uint32_t)((2 * t) * 16 + g), acc[0]);
            sts_f32(mine + 4u * (uint32_t)((2 * t + 1) * 16 + g), acc[1]);
            sts_f32(mine + 4u * (uint32_t)((2 * t) * 16 + g + 8), acc[2]);
            sts_f32(mine + 4u * (uint32_t)((2 * t + 1) * 16 + g + 8), acc[3]);
            named_bar_sync(1 + grp, 32 * ks);
            for (int o = kg * 32 + lane; o < p.n_tok * TC_ROWS; o += 32 * ks) {
                const int tok = o >> 4, row = o & 15;
                float s = 0.f;
                for (int w = 0; w < ks; ++w) s += lds_f32(pb + (uint32_t)(w * 512 + 4 * o));
                if (r0 + row < p.rows) p.y[(int64_t)tok * p.rows + r0 + row] = s;
            }
        }
    }
    // a warp that gave up waits (again bounded) for the copies it still has in
    // flight; if that wait runs out too, copies may still land in this CTA's
    // shared memory after it exits: DEVERR_DRAIN marks the device's later
    // results as suspect
    for (int j = consumed; j < issued; ++j) {
        const int sl = j % S;
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(bar0 + 8u * (uint32_t)sl, (uint32_t)((j / S) & 1)))) {
            if (lane == 0) atomicOr(p.err, DEVERR_DRAIN);
            break;
        }
    }
}

template <int FMT>
cudaError_t launch_tc(const TcParams &p, bool x_smem, dim3 grid, size_t smem, cudaStream_t st, bool pdl);

}  // namespace qmv
