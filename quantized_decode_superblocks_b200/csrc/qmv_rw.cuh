// qmv_rw.cuh -- the one-token matvec with warp-private copy rings.
//
// A batch-1 decode matvec is bound by how fast the SM can decode weights once
// the bytes stream at HBM speed (the decode costs a few instructions per
// weight, and 148 SMs must decode ~10^13 weights/s).  This kernel therefore
// spends as little as possible outside the decode itself:
//   * every warp owns a contiguous run of row groups (R rows each) and runs its
//     own ring of shared-memory stages: lane 0 moves a tile (R rows x one
//     K-chunk of up to 2048 columns) with 1-D bulk async copies that complete
//     on the stage's mbarrier, and refills the stage as soon as the warp has
//     finished with it -- no cross-warp tickets or block barriers per tile;
//   * the slice geometry is fixed at compile time: lane l decodes 64
//     consecutive-in-layout weights of every row of the tile (a pair of Q8_0
//     blocks, or a quarter of a Q4_K / Q6_K superblock) against x values that
//     sit in its registers for the whole K-chunk;
//   * one multi-row butterfly per row group reduces the lanes' partial sums.
// Decode is memory-bandwidth bound on the pages' hardware (BebeLM：纯Rust实现的
// 端侧大模型推理引擎, §性能表现); on this one the decode arithmetic is the
// tighter limit, which is what the layout above optimises for.
//
// The same body serves one matvec (one task, all CTAs) and several
// independent matvecs (each task owns a range of CTAs).
#pragma once

#include "qmv_kernels.cuh"

namespace qmv {

constexpr int RW_CK = 2048;           // columns of one K-chunk: 64 per lane
constexpr int RW_MAX_STAGES = 6;      // ring stages per warp
constexpr int RW_MAX_TASKS = 64;
constexpr int RW_CUR_OFF = 512;       // per-warp producer cursors (32 bytes each) after the mbarriers
constexpr int RW_BAR_BYTES = 1024;    // mbarriers (NW x RW_MAX_STAGES x 8 bytes) + cursors, rounded up;
                                      // the launch's task table follows (rw_hdr_bytes)
constexpr int RW_X_SMEM_MAX = 12288;  // longest row (columns) whose x is staged in shared memory

struct RwTask {
    const uint8_t *W;         // rows x row_bytes of packed blocks
    const float *x;           // [cols]
    float *y;                 // [rows]
    int64_t rows;
    int64_t row_bytes;
    int64_t n_rg;             // row groups: ceil(rows / R)
    int64_t rg_q;             // warp w = (wg - rot) mod nw of the task's nw warps takes row
    int32_t rg_r;             //   groups [w*rg_q + min(w, rg_r), +rg_q + (w < rg_r))
    int32_t rot;              // first warp of the task: consecutive small tasks land on different warps
    int32_t nw;               // warps the task is spread over
    int32_t n_chunks;         // ceil(cols / RW_CK)
    int32_t chunk_bytes;      // bytes of one full K-chunk of a row
    int32_t last_bytes;       // bytes of the last K-chunk of a row
    int32_t last_cols;        // columns of the last K-chunk
    int32_t pad_[3];
};
static_assert(sizeof(RwTask) % 16 == 0, "task table is copied in 16-byte units");

// Shared-memory header of a launch with n tasks: mbarriers, cursors, and a copy
// of the task table (read at every task switch: shared memory, not the
// constant bank, whose cache a 5 KB table with runtime indices keeps missing).
__host__ __device__ constexpr int rw_hdr_bytes(int n_tasks)
{
    return RW_BAR_BYTES + ((n_tasks * (int)sizeof(RwTask) + 127) & ~127);
}

// Launch parameters for up to NT tasks (NT = 1 keeps a single matvec's
// parameter block small: it is copied with every launch).
template <int NT>
struct RwParamsT {
    int32_t n_tasks;
    int32_t n_stage;          // ring stages per warp
    int32_t stage_pitch;      // bytes per stage (multiple of 128)
    int32_t x_floats;         // shared-memory x: the longest task row (floats), one such row per token
    int32_t cta_begin[NT + 1];   // task t owns CTAs [cta_begin[t], cta_begin[t+1])
    int *err;
    uint32_t debug_extra_tx;  // test hook: bytes expected per tile beyond those copied (0 in use)
    RwTask t[NT];
};
using RwParams1 = RwParamsT<1>;

// Row groups [a, b) of a task that warp wg takes: contiguous, balanced, split
// on the host (no divisions here).
__device__ __forceinline__ void rw_range(const RwTask &tk, int wg, int64_t &a, int64_t &b)
{
    int w = wg - tk.rot;
    if (w < 0) w += tk.nw;
    a = (int64_t)w * tk.rg_q + min(w, tk.rg_r);
    b = a + tk.rg_q + (w < tk.rg_r ? 1 : 0);
}

// The producer's position in a warp's tile sequence: task, row group, K-chunk
// (with the task's K-chunk count cached).
struct RwCursor {
    int t;
    int kc;
    int nch;
    int issued;         // tiles issued so far
    int64_t rg;
    int64_t rg_end;
};
static_assert(sizeof(RwCursor) == 32, "cursor slot");

// Move c to the first tile of task t or, if the warp has none there, of the
// next task where it has some (c.t == t_end: no tiles left).
static __device__ __noinline__ void rw_seek(const RwTask *tasks, RwCursor &c, int t, int t_end, int wg)
{
    for (; t < t_end; ++t) {
        int64_t a, b;
        rw_range(tasks[t], wg, a, b);
        if (a < b) {
            c.t = t;
            c.kc = 0;
            c.nch = tasks[t].n_chunks;
            c.rg = a;
            c.rg_end = b;
            return;
        }
    }
    c.t = t_end;
    c.kc = 0;
    c.nch = 1;
    c.rg = 0;
    c.rg_end = 0;
}

__device__ __forceinline__ void rw_advance(const RwTask *tasks, RwCursor &c, int t_end, int wg)
{
    if (++c.kc < c.nch) return;
    c.kc = 0;
    if (++c.rg < c.rg_end) return;
    rw_seek(tasks, c, c.t + 1, t_end, wg);
}

// Issue the copies of tile c into stage dst (called by one lane).
template <int R>
__device__ __forceinline__ void rw_issue(const RwTask *tasks, const RwCursor &c, uint32_t dst, uint32_t bar,
                                         uint32_t extra_tx)
{
    const RwTask &tk = tasks[c.t];
    const int64_t r0 = c.rg * R;
    const int tr = (int)min((int64_t)R, tk.rows - r0);
    const bool lastc = c.kc == c.nch - 1;
    const uint32_t cb = (uint32_t)(lastc ? tk.last_bytes : tk.chunk_bytes);
    mbar_arrive_expect_tx(bar, (uint32_t)tr * cb + extra_tx);
    const uint8_t *src = tk.W + r0 * tk.row_bytes + (int64_t)c.kc * tk.chunk_bytes;
    if (c.nch == 1) {
        bulk_g2s(dst, src, (uint32_t)tr * cb, bar);      // the tile's rows are contiguous
    } else {
        for (int k = 0; k < tr; ++k) bulk_g2s(dst + (uint32_t)k * cb, src + k * tk.row_bytes, cb, bar);
    }
}

// Two consecutive Q8_0 blocks (68 bytes at a 4-byte-aligned shared address):
// block 0's quants straddle words 0..8 (two bytes in), block 1's are words
// 9..16.  Groups gq = 0..15 of the x pairs are columns 4gq.. of the pair.
// Block 0 is finished (scaled by its d) before block 1 starts, so only two
// packed accumulators and nine words are live at a time.
template <class XP>
__device__ __forceinline__ float q8_0_dot_pair(uint32_t a, XP &&xp)
{
    float r;
    {
        uint32_t w[9];
#pragma unroll
        for (int i = 0; i < 9; ++i) w[i] = lds_u32(a + 4u * (uint32_t)i);
        float2 s0 = make_float2(0.f, 0.f), s1 = make_float2(0.f, 0.f);
#pragma unroll
        for (int gq = 0; gq < 8; ++gq) {           // bytes 2 + 4gq .. 5 + 4gq of the pair
            float2 p02, p13, x02, x13;
            bytes4_to_f2(__byte_perm(w[gq], w[gq + 1], 0x5432u) ^ 0x80808080u, 128.0f, p02, p13);
            xp(gq, x02, x13);
            s0 = f2fma(p02, x02, s0);
            s1 = f2fma(p13, x13, s1);
        }
        r = half_bits_to_float(w[0]) * hsum2(s0, s1);
    }
    const float d1 = half_bits_to_float(lds_u32(a + 32u) >> 16);
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i] = lds_u32(a + 36u + 4u * (uint32_t)i);
    float2 t0 = make_float2(0.f, 0.f), t1 = make_float2(0.f, 0.f);
#pragma unroll
    for (int gq = 0; gq < 8; ++gq) {               // aligned words 9 + gq
        float2 p02, p13, x02, x13;
        bytes4_to_f2(w[gq] ^ 0x80808080u, 128.0f, p02, p13);
        xp(8 + gq, x02, x13);
        t0 = f2fma(p02, x02, t0);
        t1 = f2fma(p13, x13, t1);
    }
    return fmaf(d1, hsum2(t0, t1), r);
}

// One token: lane l's 64-weight slice at shared address a against the x
// groups xp holds (rw_group_col order); xsa / xsb are the sums of groups 0..7
// and 8..15 (the K-quant min terms).
// PS: x holds the Q4_K groups pre-scaled by q4k_prescale_x (rw_load_x_smem<FMT, true>).
template <int FMT, bool PS = true, class XP>
__device__ __forceinline__ float lane_dot(uint32_t a, int l, const Q4kSel &sel, XP &&xp, float xsa, float xsb)
{
    if (FMT == FMT_Q8_0) return q8_0_dot_pair(a, xp);
    if (FMT == FMT_Q4_0) return q4_0_dot_pair(a, xp);
    if (FMT == FMT_Q4_K) return PS ? q4_k_dot1s(a, l & 3, sel, xp, xsa, xsb) : q4_k_dot1<false>(a, l & 3, sel, xp, xsa, xsb);
    if (FMT == FMT_Q5_K) return q5_k_dot1<false>(a, l & 3, sel, xp, xsa, xsb);
    return q6_k_dot1(a, (l >> 1) & 1, 16 * (l & 1), xp);
}

// Column (within the K-chunk) of x group gq of lane l's 64-weight slice.
template <int FMT>
__device__ __forceinline__ int rw_group_col(int l, int gq)
{
    if (small_block<FMT>()) return 64 * l + 4 * gq;
    return slice1_group_col<FMT>(l, gq);
}

// Byte offset of lane l's 64-weight slice within a row: two 32-weight blocks,
// or a quarter of a superblock.
template <int FMT>
__device__ __forceinline__ uint32_t lane_slice_off(int l)
{
    if (small_block<FMT>()) return 2u * (uint32_t)Fmt<FMT>::BB * (uint32_t)l;
    return (uint32_t)Fmt<FMT>::BB * (uint32_t)(l >> 2);
}

// Shared address of lane l's slice within one row of a stage.
template <int FMT>
__device__ __forceinline__ uint32_t rw_slice_addr(uint32_t rowp, int l)
{
    return rowp + lane_slice_off<FMT>(l);
}

// A task's x sits in shared memory for the whole task; a lane loads its 64
// values of a K-chunk into registers from there (once per task for rows of
// one K-chunk, once per tile for longer rows).  float4 f of the row is stored
// at f ^ ((f >> 4) & 7): the eight lanes of a quarter-warp that read the same
// group of their 64-column slices hit eight different bank groups.  Chained
// launches read x through L2 only: it may have been written by another SM
// earlier in the same launch.
__device__ __forceinline__ uint32_t rw_xswz(uint32_t f) { return f ^ ((f >> 4) & 7u); }

__device__ __forceinline__ void rw_stage_x(uint32_t xs, const float *x, int cols, bool coherent)
{
    for (int f = (int)threadIdx.x; f < (cols >> 2); f += NTHREADS) {
        const float4 *src = reinterpret_cast<const float4 *>(x) + f;
        sts_f4(xs + 16u * rw_xswz((uint32_t)f), coherent ? __ldcg(src) : __ldg(src));
    }
}

template <int FMT, bool PS = true>
__device__ __forceinline__ void rw_load_x_smem(uint32_t xs, int kc, int ncols, int lane, float2 (&xr)[16][2],
                                               float &xsa, float &xsb)
{
    const bool have = 64 * (lane + 1) <= ncols;
    float2 sa = make_float2(0.f, 0.f), sb = make_float2(0.f, 0.f);
#pragma unroll
    for (int gq = 0; gq < 16; ++gq) {
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (have) v = lds_f4(xs + 16u * rw_xswz((uint32_t)((kc * RW_CK + rw_group_col<FMT>(lane, gq)) >> 2)));
        xr[gq][0] = make_float2(v.x, v.z);
        xr[gq][1] = make_float2(v.y, v.w);
        if (gq < 8) sa = f2add(sa, f2add(xr[gq][0], xr[gq][1]));
        else sb = f2add(sb, f2add(xr[gq][0], xr[gq][1]));
    }
    xsa = sa.x + sa.y;
    xsb = sb.x + sb.y;
    if (FMT == FMT_Q4_K && PS) q4k_prescale_x(xr);     // the groups lane_dot<FMT, true> expects
}

// Accumulators of one row group: one token -> a float per row (factored
// decode); several tokens -> a packed pair per (row, token) (weight-stationary
// decode units of qmv_decodemt.cuh).
template <int R, int NTOK> struct RwAcc {
    float2 v[R][NTOK];
    __device__ __forceinline__ void zero()
    {
#pragma unroll
        for (int k = 0; k < R; ++k)
#pragma unroll
            for (int t = 0; t < NTOK; ++t) v[k][t] = make_float2(0.f, 0.f);
    }
};
template <int R> struct RwAcc<R, 1> {
    float v[R];
    __device__ __forceinline__ void zero()
    {
#pragma unroll
        for (int k = 0; k < R; ++k) v[k] = 0.f;
    }
};

// Three or more tokens: one CTA per SM, with the SM's whole shared memory
// (every token's x) and registers (the accumulators) -- no spills.
template <int FMT, int R, int NT, int NTOK>
__global__ void __launch_bounds__(NTHREADS, (NTOK > 2 ? 1 : 2)) qmv_rw_kernel(const __grid_constant__ RwParamsT<NT> p)
{
    static_assert(R == 1 || R == 2 || R == 4 || R == 8, "R");
    static_assert(NTOK >= 1 && NTOK <= 8 && (NTOK == 1 || NT == 1), "several tokens: single launches only");
    constexpr int NTP = Pow2Ceil<NTOK>::v;
    static_assert(R * NTP <= 32, "R * n_tok too large for one warp reduction");
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = (int)threadIdx.x >> 5, lane = (int)threadIdx.x & 31;
    const uint32_t sraw = smem_addr(smem);
    const uint32_t sbase = (sraw + 127u) & ~127u;          // the launch adds 128 spare bytes
    const int S = p.n_stage;
    const uint32_t full0 = sbase + 8u * (uint32_t)(warp * RW_MAX_STAGES);
    RwTask *const tasks = reinterpret_cast<RwTask *>(smem + (sbase - sraw) + RW_BAR_BYTES);
    const uint32_t xs = sbase + (uint32_t)rw_hdr_bytes(p.n_tasks);
    const uint32_t x_area = (uint32_t)NTOK * (uint32_t)(((p.x_floats * 4) + 127) & ~127);   // one row per token
    const uint32_t stage0 = xs + x_area + (uint32_t)(warp * S) * (uint32_t)p.stage_pitch;

    int tt = 0;
    while (tt + 1 < p.n_tasks && (int)blockIdx.x >= p.cta_begin[tt + 1]) ++tt;
    const int t_begin = tt, t_end = tt + 1;
    const int wg = ((int)blockIdx.x - p.cta_begin[tt]) * NW + warp;

    {
        const uint4 *src = reinterpret_cast<const uint4 *>(&p.t[0]);
        uint4 *dst = reinterpret_cast<uint4 *>(tasks);
        for (int i = (int)threadIdx.x; i < p.n_tasks * (int)(sizeof(RwTask) / 16); i += NTHREADS) dst[i] = src[i];
    }
    if (lane == 0) {
        for (int s = 0; s < S; ++s) mbar_init(full0 + 8u * (uint32_t)s, 1);
        fence_mbar_init();
    }
    __syncthreads();
    pdl_launch_dependents();

    // The producer cursor lives in shared memory and only lane 0 touches it
    // (keeps the consumer's registers for x and the decode).
    RwCursor *const cur = reinterpret_cast<RwCursor *>(smem + (sbase - sraw) + RW_CUR_OFF) + warp;
    // prologue: the first S tiles (weights only: no dependence on earlier kernels)
    if (lane == 0) {
        RwCursor f;
        rw_seek(tasks, f, t_begin, t_end, wg);
        f.issued = 0;
        for (int s = 0; s < S && f.t < t_end; ++s) {
            rw_issue<R>(tasks, f, stage0 + (uint32_t)s * (uint32_t)p.stage_pitch, full0 + 8u * (uint32_t)s,
                        p.debug_extra_tx);
            rw_advance(tasks, f, t_end, wg);
            ++f.issued;
        }
        *cur = f;
    }
    int consumed = 0;

    pdl_wait();                                    // x is the previous kernel's output
    const Q4kSel sel = q4k_sel(lane & 3);
    bool dead = false;
    int slot = 0;
    uint32_t phase = 0;
    const uint32_t pitch = (uint32_t)p.stage_pitch;

    float2 xr[16][2];
    float xsa = 0.f, xsb = 0.f;
    for (int t = t_begin; t < t_end; ++t) {
        const RwTask &tk = tasks[t];
        const int nch = tk.n_chunks;
        // The CTA copies the task's x into shared memory once (every thread a
        // few float4s) and every warp takes its slices from there: one 8 KB
        // read per CTA from L2 instead of one per warp, which matters because
        // those L2 reads queue behind the weight copies in flight.
        const int cols_t = (nch - 1) * RW_CK + tk.last_cols;
        const uint32_t xrow = (uint32_t)((cols_t * 4 + 127) & ~127);   // bytes per token row of staged x
#pragma unroll 1
        for (int n = 0; n < NTOK; ++n) rw_stage_x(xs + (uint32_t)n * xrow, tk.x + (int64_t)n * cols_t, cols_t, false);
        __syncthreads();
        int64_t a, b;
        rw_range(tk, wg, a, b);
        if (a >= b || dead) {
            __syncthreads();                      // matches the one after the task below
            continue;
        }
        // the task's fields, once
        float *ty = tk.y;
        const int64_t rows = tk.rows;
        const int last_cols = tk.last_cols;
        const uint32_t last_bytes = (uint32_t)tk.last_bytes;
        const uint32_t chunk_bytes = (uint32_t)tk.chunk_bytes;
        // one tile: wait for the stage, decode R rows of it, hand the stage back
        // to the producer (refilled with the tile S ahead)
        auto tile = [&](RwAcc<R, NTOK> &acc, int ncols, uint32_t cb, int kc) -> bool {
            const uint32_t full = full0 + 8u * (uint32_t)slot;
            // every lane times its own wait: agree on the outcome so the warp stays converged
            if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(full, phase))) {
                if (lane == 0) atomicOr(p.err, DEVERR_TIMEOUT);
                return false;
            }
            ++consumed;
            const uint32_t st = stage0 + (uint32_t)slot * pitch;
            if (64 * (lane + 1) <= ncols) {
                if constexpr (NTOK == 1) {
                    auto xp = [&](int gq, float2 &x02, float2 &x13) {
                        x02 = xr[gq][0];
                        x13 = xr[gq][1];
                    };
                    uint32_t sa = rw_slice_addr<FMT>(st, lane);
#pragma unroll
                    for (int k = 0; k < R; ++k, sa += cb) {
                        acc.v[k] += lane_dot<FMT, false>(sa, lane, sel, xp, xsa, xsb);
                    }
                } else {
                    // several tokens: weights decoded once per step, each token's
                    // x (staged, swizzled) spent on all R rows
                    auto xl = [&](int n, int col) {
                        return lds_f4(xs + (uint32_t)n * xrow + 16u * rw_xswz((uint32_t)col >> 2));
                    };
                    const int cbase = kc * RW_CK;
                    uint32_t bp[R];
                    if (FMT == FMT_Q8_0) {
#pragma unroll
                        for (int b = 0; b < 2; ++b) {
#pragma unroll
                            for (int k = 0; k < R; ++k) bp[k] = st + (uint32_t)k * cb + 68u * (uint32_t)lane + 34u * (uint32_t)b;
                            q8_0_slice_mt<NTOK, R>(bp, cbase + 64 * lane + 32 * b, xl, acc.v);
                        }
                    } else if (FMT == FMT_Q4_K) {
#pragma unroll
                        for (int k = 0; k < R; ++k) bp[k] = st + (uint32_t)k * cb + 144u * (uint32_t)(lane >> 2);
                        q4_k_slice_mt<NTOK, R>(bp, lane & 3, sel, cbase + 64 * lane, xl, acc.v);
                    } else {
#pragma unroll
                        for (int k = 0; k < R; ++k) bp[k] = st + (uint32_t)k * cb + 210u * (uint32_t)(lane >> 2);
                        const int h = (lane >> 1) & 1, l0 = 16 * (lane & 1);
                        q6_k_slice_mt<NTOK, R>(bp, h, l0, cbase + 256 * (lane >> 2) + 128 * h + l0, xl, acc.v);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) {
                RwCursor f = *cur;
                if (f.t < t_end) {
                    fence_proxy_async_smem();
                    rw_issue<R>(tasks, f, st, full, p.debug_extra_tx);
                    rw_advance(tasks, f, t_end, wg);
                    ++f.issued;
                    *cur = f;
                }
            }
            if (++slot == S) {
                slot = 0;
                phase ^= 1u;
            }
            return true;
        };
        auto finish = [&](RwAcc<R, NTOK> &acc, int64_t rg) {
            constexpr int V = R * NTP;
            float vals[V];
#pragma unroll
            for (int k = 0; k < R; ++k)
#pragma unroll
                for (int n = 0; n < NTP; ++n) {
                    if constexpr (NTOK == 1) vals[k] = acc.v[k];
                    else vals[k * NTP + n] = n < NTOK ? acc.v[k][n < NTOK ? n : 0].x + acc.v[k][n < NTOK ? n : 0].y : 0.f;
                }
            warp_transpose_reduce<V>(vals, lane);
            constexpr int SH = 5 - Log2<V>::v;
            const int idx = lane >> SH, k = idx / NTP, n = idx % NTP;
            const int64_t row = rg * R + k;
            if ((lane & ((1 << SH) - 1)) == 0 && n < NTOK && row < rows) ty[(int64_t)n * rows + row] = vals[0];
        };
        if (nch == 1) {
            // one token: x stays in registers for the whole task
            if constexpr (NTOK == 1) rw_load_x_smem<FMT, false>(xs, 0, last_cols, lane, xr, xsa, xsb);
            for (int64_t rg = a; rg < b; ++rg) {
                RwAcc<R, NTOK> acc;
                acc.zero();
                if (!tile(acc, last_cols, last_bytes, 0)) {
                    dead = true;
                    break;
                }
                finish(acc, rg);
            }
        } else {
            for (int64_t rg = a; rg < b && !dead; ++rg) {
                RwAcc<R, NTOK> acc;
                acc.zero();
                for (int kc = 0; kc < nch; ++kc) {
                    const bool lastc = kc == nch - 1;
                    const int ncols = lastc ? last_cols : RW_CK;
                    if constexpr (NTOK == 1) rw_load_x_smem<FMT, false>(xs, kc, ncols, lane, xr, xsa, xsb);
                    if (!tile(acc, ncols, lastc ? last_bytes : chunk_bytes, kc)) {
                        dead = true;
                        break;
                    }
                }
                if (!dead) finish(acc, rg);
            }
        }
        __syncthreads();                          // x stays until every warp is done with it
    }
    // after a timeout: let the copies still in flight land before the CTA
    // exits; if that wait runs out too, DEVERR_DRAIN marks the device's later
    // results as suspect (copies may land in shared memory after the exit)
    if (dead) {
        int pending = __shfl_sync(0xFFFFFFFFu, lane == 0 ? cur->issued : 0, 0) - consumed;
        for (; pending > 0; --pending) {
            if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(full0 + 8u * (uint32_t)slot, phase))) {
                if (lane == 0) atomicOr(p.err, DEVERR_DRAIN);
                break;
            }
            if (++slot == S) {
                slot = 0;
                phase ^= 1u;
            }
        }
    }
}

// Defined per format in qmv_fmt_*.cu.
template <int FMT, int NT>
cudaError_t launch_rw(const RwParamsT<NT> &p, int R, dim3 grid, size_t smem, cudaStream_t stream, bool pdl,
                      bool cooperative);
// Several tokens (2..4), single launches (3 and 4: one CTA per SM).
template <int FMT>
cudaError_t launch_rw_mt(const RwParams1 &p, int n_tok, int R, dim3 grid, size_t smem, cudaStream_t stream, bool pdl);

}  // namespace qmv
