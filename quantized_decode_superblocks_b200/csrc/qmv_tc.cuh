// qmv_tc.cuh -- several-token (3..8) Q8_0 matvec on the tensor cores.
//
// With n_tok tokens every weight feeds n_tok products; on the CUDA cores that
// is n_tok FMAs plus n_tok x reads per weight, which made the 8-token decode
// step six times slower than the 1-token one.  Here the weights of a tile of
// 16 rows are decoded exactly (Q8_0 quants are small integers, exact in
// TF32) straight into the A fragments of mma.m16n8k8 (TF32 in, f32
// accumulate) and the tokens form the N = 8 columns.  x is split as
// hi = tf32(x), lo = x - hi: two MMAs per k-step keep the products within
// about 2^-21 of f32 (TF32 alone would lose 11 bits of x).  Each 32-column
// block's sum is scaled by its f32 d in registers (GGUF Q8_0 layout: one fp16
// d and 32 int8 quants per block; dequantized weight d * q), so only
// integers go through the tensor cores.
//
// Data flow: one CTA per SM (16 warps); the CTA's x rows sit in shared
// memory (token-major, row pitch cols + 4 floats so a warp's 16-byte loads
// hit all banks once) or, when they do not fit next to the rings, are read
// through L2.  A unit is one tile (16 rows x 256 columns = 4352 bytes),
// copied by `cp.async.bulk` (one copy per row) into a warp-private ring of
// stages on an mbarrier, as in the warp-ring kernel.  The CTA's row tiles go
// to groups of `ksplit` warps; the warps of a group split the K-chunks of a
// tile, add their partial sums in a fixed order through shared memory
// (named barrier per group) and write y.
#pragma once

#include "qmv_kernels.cuh"

namespace qmv {

constexpr int TC_KCOLS = 256;          // columns per K-chunk (a multiple of 16 bytes in Q8_0)
constexpr int TC_ROWS = 16;            // rows per tile (MMA M)
constexpr int TC_MAX_STAGES = 6;
constexpr int TC_WARPS = 16;           // warps per CTA (one CTA per SM)
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
    int32_t chunk_bytes;   // bytes of one row's K-chunk
    int32_t ksplit;        // warps per row-tile group (divides TC_NW and kc_n)
    int32_t n_rt;          // row tiles in the matrix
    int32_t rt_q, rt_r;    // CTA c owns rt_q + (c < rt_r) consecutive row tiles
    int32_t n_stage;       // ring stages per warp
    int32_t x_pitch;       // floats per token row of shared x (cols + 4)
    int *err;
};

__host__ __device__ constexpr uint32_t tc_round128(uint32_t b) { return (b + 127u) & ~127u; }

// Round-to-nearest TF32 of v, as a 32-bit pattern with the low 13 bits clear.
__device__ __forceinline__ uint32_t tf32_rna(float v)
{
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(v));
    return r;
}

// d[0..3] += A (16x8, TF32) * B (8x8, TF32), f32 accumulation.  Fragments as
// the PTX ISA defines them for m16n8k8 (g = lane / 4, t = lane % 4):
// a0 (g, t), a1 (g + 8, t), a2 (g, t + 4), a3 (g + 8, t + 4);
// b0 (k = t, n = g), b1 (k = t + 4, n = g);
// d0 (g, 2t), d1 (g, 2t + 1), d2 (g + 8, 2t), d3 (g + 8, 2t + 1).
__device__ __forceinline__ void mma_tf32(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1)
{
    asm("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 "
                 "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

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

// x[token g][32b + 8t .. + 7] of block b as TF32 hi / lo halves (B fragments),
// from shared memory (XS; xrow a shared address) or through L2 (xg).
template <bool XS>
__device__ __forceinline__ void tc_x_frag(uint32_t xrow, const float *xg, int b, int t, bool have_x,
                                          uint32_t (&bh)[8], uint32_t (&bl)[8])
{
    float4 xa = make_float4(0.f, 0.f, 0.f, 0.f), xb = xa;
    if (have_x) {
        if (XS) {
            xa = lds_f4(xrow + 4u * (uint32_t)(32 * b + 8 * t));
            xb = lds_f4(xrow + 4u * (uint32_t)(32 * b + 8 * t + 4));
        } else {
            xa = __ldg(reinterpret_cast<const float4 *>(xg + 32 * b + 8 * t));
            xb = __ldg(reinterpret_cast<const float4 *>(xg + 32 * b + 8 * t + 4));
        }
    }
    const float xv[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        bh[i] = tf32_rna(xv[i]);
        bl[i] = __float_as_uint(xv[i] - __uint_as_float(bh[i]));
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

// One 16 x 256 Q8_0 tile against the 8 token columns: acc (rows g, g + 8;
// tokens 2t, 2t + 1) += sum over the 8 blocks of d_row * (q . x).
// Column map: the k-step s of block b gives thread t the columns
// 32b + 8t + 2s (logical k = t) and 32b + 8t + 2s + 1 (k = t + 4), on both
// the A and the B side, so a thread's A bytes and x values are 8 consecutive
// columns.  Two blocks at a time, each with separate hi and lo accumulators:
// four independent MMA chains of four, so a warp does not wait out the MMA
// latency at every step.
template <int B0, bool XS>
__device__ __forceinline__ void tc_q8_pair(uint32_t ra, uint32_t rb, uint32_t xrow, const float *xg, bool have_x, int t,
                                           float (&acc)[4])
{
    uint32_t h0[8], l0[8], h1[8], l1[8];
    tc_x_frag<XS>(xrow, xg, B0, t, have_x, h0, l0);
    tc_x_frag<XS>(xrow, xg, B0 + 1, t, have_x, h1, l1);
    float q0[16], q1[16];
    tc_q8_frag<B0>(ra, rb, t, q0);
    tc_q8_frag<B0 + 1>(ra, rb, t, q1);
    float c0h[4] = {0.f, 0.f, 0.f, 0.f}, c0l[4] = {0.f, 0.f, 0.f, 0.f};
    float c1h[4] = {0.f, 0.f, 0.f, 0.f}, c1l[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        const uint32_t a0 = __float_as_uint(q0[2 * s]), a2 = __float_as_uint(q0[2 * s + 1]);
        const uint32_t a1 = __float_as_uint(q0[8 + 2 * s]), a3 = __float_as_uint(q0[8 + 2 * s + 1]);
        const uint32_t e0 = __float_as_uint(q1[2 * s]), e2 = __float_as_uint(q1[2 * s + 1]);
        const uint32_t e1 = __float_as_uint(q1[8 + 2 * s]), e3 = __float_as_uint(q1[8 + 2 * s + 1]);
        mma_tf32(c0h, a0, a1, a2, a3, h0[2 * s], h0[2 * s + 1]);
        mma_tf32(c1h, e0, e1, e2, e3, h1[2 * s], h1[2 * s + 1]);
        mma_tf32(c0l, a0, a1, a2, a3, l0[2 * s], l0[2 * s + 1]);
        mma_tf32(c1l, e0, e1, e2, e3, l1[2 * s], l1[2 * s + 1]);
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

template <bool XS>
__device__ __forceinline__ void tc_q8_tile(uint32_t st, int chunk_bytes, uint32_t xrow, const float *xg, bool have_x,
                                           int g, int t, float (&acc)[4])
{
    const uint32_t ra = st + (uint32_t)(g * chunk_bytes);
    const uint32_t rb = ra + 8u * (uint32_t)chunk_bytes;
    tc_q8_pair<0, XS>(ra, rb, xrow, xg, have_x, t, acc);
    tc_q8_pair<2, XS>(ra, rb, xrow, xg, have_x, t, acc);
    tc_q8_pair<4, XS>(ra, rb, xrow, xg, have_x, t, acc);
    tc_q8_pair<6, XS>(ra, rb, xrow, xg, have_x, t, acc);
}

template <int FMT, int NWARP, bool XS>
__global__ void __launch_bounds__(NWARP * 32, 1) qmv_tc_kernel(const TcParams p)
{
    constexpr int TC_NW = NWARP;
    constexpr int TC_NT = NWARP * 32;
    constexpr int TC_PART_BYTES = tc_part_bytes(NWARP);
    static_assert(FMT == FMT_Q8_0, "tensor-core path: Q8_0");
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
    const uint32_t tile_bytes = (uint32_t)(TC_ROWS * p.chunk_bytes);
    const uint32_t stage0 = part + (uint32_t)TC_PART_BYTES + (uint32_t)(warp * S) * tile_bytes;

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
        if (lane == 0) mbar_arrive_expect_tx(bar, (uint32_t)(valid * p.chunk_bytes));
        __syncwarp();
        if (lane < valid)
            bulk_g2s(stage0 + (uint32_t)sl * tile_bytes + (uint32_t)(lane * p.chunk_bytes),
                     p.W + (r0 + lane) * p.row_bytes + (int64_t)kc * p.chunk_bytes, (uint32_t)p.chunk_bytes, bar);
    };
    int issued = 0;
    for (; issued < S && issued < n_units; ++issued) issue(issued);   // weights: no dependence on earlier kernels

    pdl_wait();                                         // x is the previous kernel's output
    if (XS) {
        const int c4 = p.cols >> 2;
        for (int i = (int)threadIdx.x; i < p.n_tok * c4; i += TC_NT) {
            const int tok = i / c4, f = i - tok * c4;
            const float4 v = __ldg(reinterpret_cast<const float4 *>(p.x + (int64_t)tok * p.cols) + f);
            sts_f4(xs + 4u * (uint32_t)(tok * p.x_pitch + 4 * f), v);
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
                    tc_q8_tile<XS>(stage0 + (uint32_t)sl * tile_bytes, p.chunk_bytes,
                                   xrow0 + 4u * (uint32_t)(kc * TC_KCOLS), xg0 + kc * TC_KCOLS, have_x, g, t, acc);
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
    // a warp that gave up waits (again bounded) for the copies it still has in flight
    for (int j = consumed; j < issued; ++j) {
        const int sl = j % S;
        (void)mbar_wait_bounded(bar0 + 8u * (uint32_t)sl, (uint32_t)((j / S) & 1));
    }
}

template <int FMT>
cudaError_t launch_tc(const TcParams &p, bool x_smem, dim3 grid, size_t smem, cudaStream_t st, bool pdl);

}  // namespace qmv
