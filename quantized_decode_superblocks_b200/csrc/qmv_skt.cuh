// qmv_skt.cuh -- the streaming matvec for a few tokens (speculative
// verification, FlareLLM：纯Rust打造的浏览器端LLM推理引擎, §推理层面的深度优化:
// several tokens checked in one pass over the weights).
//
// The same producer warp, ring of whole-row stages and consumer split as the
// one-token streaming kernel (qmv_sk.cuh); what changes is the consumer's
// arithmetic.  Every token's x stays in shared memory (n_tok rows, swizzled
// as for one token) instead of in registers, and the decode runs the
// weight-stationary units of qmv_decodemt.cuh: a few weights of each of the
// warp's R rows are decoded once into exact f32 (scales applied), then each
// token's x for those columns is read once and spent on all R rows.  A lane
// still owns 64 layout-consecutive weights of every row of its K-segment.
// Rows of a row slot past the matrix end are decoded from the slot's first
// row and never stored.
#pragma once

#include "qmv_sk.cuh"

namespace qmv {

constexpr int SKT_MAX_NTOK = 4;

// The x rows of n_tok tokens into the swizzled x area, token t at byte
// t * x_row: all of a thread's loads of a pass in flight before its stores.
__device__ __forceinline__ void skt_stage_x(uint32_t xs, const float *x, int n_tok, int nr, int cols, int x_row)
{
    constexpr int B = 8;
    const int n = n_tok * nr;
#pragma unroll 1
    for (int base = 0; base < n; base += B * SK_NC * 32) {
        float4 v[B];
#pragma unroll
        for (int j = 0; j < B; ++j) {
            const int d = base + (int)threadIdx.x + j * SK_NC * 32;
            if (d < n) {
                const int t = d / nr, c = d - t * nr;
                v[j] = __ldg(reinterpret_cast<const float4 *>(x + (int64_t)t * cols) + c);
            }
        }
#pragma unroll
        for (int j = 0; j < B; ++j) {
            const int d = base + (int)threadIdx.x + j * SK_NC * 32;
            if (d < n) {
                const int t = d / nr, c = d - t * nr;
                sts_f4(xs + (uint32_t)(t * x_row) + 16u * rw_xswz((uint32_t)c), v[j]);
            }
        }
    }
}

// Lane l's 64-weight slice of the R rows at shared addresses rowp[k] (the
// rows' starts in the stage, K-segment included) against NTOK tokens' x:
// acc[k][t] += the slice's part of row k . x_t.  col0 = the slice's first
// column within the K-segment (64 l).
template <int FMT, int NTOK, int R, class XL>
__device__ __forceinline__ void lane_slice_mt(const uint32_t (&rowp)[R], int l, const Q4kSel &sel, XL &&xl,
                                              float2 (&acc)[R][NTOK])
{
    const int col0 = 64 * l;
    uint32_t bp[R];
    if (FMT == FMT_Q8_0 || FMT == FMT_Q4_0) {
        constexpr uint32_t BB = (uint32_t)Fmt<FMT>::BB;
#pragma unroll
        for (int b = 0; b < 2; ++b) {          // the lane's two 32-weight blocks
#pragma unroll
            for (int k = 0; k < R; ++k) bp[k] = rowp[k] + (2u * (uint32_t)l + (uint32_t)b) * BB;
            if (FMT == FMT_Q8_0) q8_0_slice_mt<NTOK, R>(bp, col0 + 32 * b, xl, acc);
            else q4_0_slice_mt<NTOK, R>(bp, col0 + 32 * b, xl, acc);
        }
    } else {
        constexpr uint32_t BB = (uint32_t)Fmt<FMT>::BB;
#pragma unroll
        for (int k = 0; k < R; ++k) bp[k] = rowp[k] + BB * (uint32_t)(l >> 2);
        if (FMT == FMT_Q4_K) {
            q4_k_slice_mt<NTOK, R>(bp, l & 3, sel, col0, xl, acc);
        } else if (FMT == FMT_Q5_K) {
            q5_k_slice_mt<NTOK, R>(bp, l & 3, sel, col0, xl, acc);
        } else {
            const int h = (l >> 1) & 1, l0 = 16 * (l & 1);
            q6_k_slice_mt<NTOK, R>(bp, h, l0, 256 * (l >> 2) + 128 * h + l0, xl, acc);
        }
    }
}

template <int FMT, int R, int NTOK>
__global__ void __launch_bounds__(SK_THREADS, 1) qmv_skt_kernel(const __grid_constant__ SkParams p)
{
    static_assert(R == 1 || R == 2 || (R == 4 && NTOK == 2), "rows per consumer warp (four: two tokens)");
    static_assert(NTOK >= 2 && NTOK <= SKT_MAX_NTOK, "tokens");
    constexpr int NTP = Pow2Ceil<NTOK>::v;
    constexpr int V = R * NTP;                    // values a warp reduces per stage: (row, token)
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = (int)threadIdx.x >> 5, lane = (int)threadIdx.x & 31;
    const uint32_t sraw = smem_addr(smem);
    const uint32_t sbase = (sraw + 127u) & ~127u;          // the launch adds 128 spare bytes
    uint8_t *const sgen = smem + (sbase - sraw);
    const uint32_t full0 = sbase + SK_FULL_OFF, empty0 = sbase + SK_EMPTY_OFF, xdone = sbase + SK_XDONE_OFF;
    volatile int *const abort_flag = reinterpret_cast<volatile int *>(sgen + SK_ABORT_OFF);
    const uint32_t part0 = sbase + (uint32_t)SK_HDR;
    const uint32_t ring = part0 + (uint32_t)SK_PART;
    const int S = p.n_stage;
    const uint32_t pitch = (uint32_t)p.stage_pitch;
    const uint32_t xs = ring + (uint32_t)p.x_off;          // x stays after the ring for the whole kernel
    auto full_bar = [&](int s) { return full0 + 8u * (uint32_t)s; };

    // this CTA's rows
    const int c = (int)blockIdx.x;
    const int64_t u0 = (int64_t)c * p.units_q + min(c, p.units_r);
    const int64_t r_begin = u0 * p.gran;
    const int64_t r_end = min(p.rows, (u0 + p.units_q + (c < p.units_r ? 1 : 0)) * p.gran);
    const int T = p.tile_rows;
    const int n_st = r_end > r_begin ? (int)((r_end - r_begin + T - 1) / T) : 0;
    const uint64_t rbw = (uint64_t)p.row_bytes;
    const uint64_t wpol = l2_evict_first_policy();
    auto issue = [&](int i, int slot) {             // stage i: one copy of T whole rows
        const int64_t r0 = r_begin + (int64_t)i * T;
        const uint32_t bytes = (uint32_t)min((int64_t)T, r_end - r0) * (uint32_t)rbw;
        mbar_arrive_expect_tx(full_bar(slot), bytes + p.debug_extra_tx);
        bulk_g2s_hint(ring + (uint32_t)slot * pitch, p.W + (uint64_t)r0 * rbw, bytes, full_bar(slot), wpol);
    };

    // barriers and a head start of weights before the CTA barrier (they
    // depend on no earlier kernel); x on its way into L2 meanwhile
    int pre = 0;
    if (warp == SK_NC && lane == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty0 + 8u * (uint32_t)s, SK_NC);
        }
        mbar_init(xdone, SK_NC);
        *abort_flag = 0;
        fence_mbar_init();
        pre = min(n_st, min(S, SK_HEAD_START));
        for (int i = 0; i < pre; ++i) issue(i, i);
    } else if (threadIdx.x == 0) {
        prefetch_l2(p.x, (uint32_t)(NTOK * p.cols * 4));
    }
    __syncthreads();
    pdl_launch_dependents();

    if (warp == SK_NC) {
        // ------------------------------------------------------ producer --
        if (lane != 0) return;
        int issued = pre;
        bool ok = true;
        for (int i = pre; i < n_st && ok; ++i) {
            const int slot = i % S;
            const int round = i / S;
            // the rest of the ring once x is in shared memory
            if (i == pre && !mbar_wait_bounded_block(xdone, 0u)) {
                atomicOr(p.err, DEVERR_TIMEOUT);
                break;
            }
            if (round > 0) ok = mbar_wait_bounded_block(empty0 + 8u * (uint32_t)slot, (uint32_t)((round - 1) & 1));
            if (!ok) {
                atomicOr(p.err, DEVERR_TIMEOUT);
                break;
            }
            if (*abort_flag) break;
            if (round > 0) fence_proxy_async_smem();   // the slot was last read through the generic proxy
            issue(i, slot);
            ++issued;
        }
        for (int i = max(0, issued - S); i < issued; ++i) {
            if (!mbar_wait_bounded_block(full_bar(i % S), (uint32_t)((i / S) & 1))) {
                atomicOr(p.err, DEVERR_DRAIN);
                break;
            }
        }
        return;
    }

    // -------------------------------------------------------- consumers --
    pdl_wait();                                    // x comes from earlier kernels
    skt_stage_x(xs, p.x, NTOK, p.cols >> 2, p.cols, p.x_row);
    named_bar_sync(1, SK_NC * 32);
    __syncwarp();
    if (lane == 0) mbar_arrive(xdone);             // x is staged: the producer may fill the rest of the ring

    const int ks = warp % p.ksegs, rs = warp / p.ksegs;
    const int seg_cols = min(SK_SEG, p.cols - ks * SK_SEG);
    const bool have = 64 * (lane + 1) <= seg_cols;
    const Q4kSel sel = q4k_sel(lane & 3);
    const uint32_t rb = (uint32_t)p.row_bytes;
    const uint32_t seg_off = (uint32_t)ks * (uint32_t)p.seg_bytes;
    const int xcol0 = ks * SK_SEG;
    auto xl = [&](int t, int col) {
        return lds_f4(xs + (uint32_t)(t * p.x_row) + 16u * rw_xswz((uint32_t)(xcol0 + col) >> 2));
    };
    constexpr int SH = 5 - Log2<V>::v;
    const bool leader = (lane & ((1 << SH) - 1)) == 0;
    const int vk = (lane >> SH) / NTP, vt = (lane >> SH) % NTP;   // (row, token) a leader holds

    bool dead = false;
    int slot = 0;
    uint32_t phase = 0;
    int64_t r0 = r_begin;
    for (int i = 0; i < n_st; ++i) {
        const uint32_t st = ring + (uint32_t)slot * pitch;
        const int ra = min(R, (int)min((int64_t)T, r_end - r0) - rs * R);     // rows of this row slot
        if (ra > 0 && !dead && !__all_sync(0xFFFFFFFFu, mbar_wait_bounded_block(full_bar(slot), phase))) {
            if (lane == 0) {
                atomicOr(p.err, DEVERR_TIMEOUT);
                *abort_flag = 1;
            }
            dead = true;                          // no more waits; stages are still released
        }
        float2 acc[R][NTOK];
#pragma unroll
        for (int k = 0; k < R; ++k)
#pragma unroll
            for (int t = 0; t < NTOK; ++t) acc[k][t] = make_float2(0.f, 0.f);
        if (!dead && ra > 0 && have) {
            uint32_t rowp[R];
#pragma unroll
            for (int k = 0; k < R; ++k)
                rowp[k] = st + (uint32_t)(rs * R + (k < ra ? k : 0)) * rb + seg_off;
            lane_slice_mt<FMT, NTOK, R>(rowp, lane, sel, xl, acc);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8u * (uint32_t)slot);   // the stage may be refilled
        float v[V];
#pragma unroll
        for (int k = 0; k < R; ++k)
#pragma unroll
            for (int t = 0; t < NTP; ++t) v[k * NTP + t] = t < NTOK ? acc[k][t].x + acc[k][t].y : 0.f;
        warp_transpose_reduce<V>(v, lane);
        const int64_t row = r0 + rs * R + vk;
        if (p.ksegs == 1) {
            if (leader && vt < NTOK && vk < ra) p.y[(int64_t)vt * p.rows + row] = v[0];
        } else {
            // partials of the row's K-segments, added in K order by segment 0
            const uint32_t pb = part0 + (uint32_t)(i & 1) * (uint32_t)(SK_PART / 2);
            const int nk = p.ksegs;
            if (leader) sts_f32(pb + 4u * (uint32_t)(((rs * R + vk) * NTP + vt) * nk + ks), v[0]);
            named_bar_sync(2 + rs, 32 * nk);
            if (ks == 0 && leader && vt < NTOK && vk < ra) {
                float s0 = 0.f;
                const uint32_t e0 = pb + 4u * (uint32_t)(((rs * R + vk) * NTP + vt) * nk);
                for (int k2 = 0; k2 < nk; ++k2) s0 += lds_f32(e0 + 4u * (uint32_t)k2);
                p.y[(int64_t)vt * p.rows + row] = s0;
            }
        }
        if (++slot == S) {
            slot = 0;
            phase ^= 1u;
        }
        r0 += T;
    }
}

// Defined per format in qmv_fmt_*.cu.
template <int FMT>
cudaError_t launch_skt(const SkParams &p, int n_tok, int R, dim3 grid, size_t smem, cudaStream_t stream, bool pdl);

}  // namespace qmv
