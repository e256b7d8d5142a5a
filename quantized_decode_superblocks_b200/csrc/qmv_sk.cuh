// qmv_sk.cuh -- the one-token streaming matvec: one producer warp, twelve
// consumer warps, whole multi-row stages.
//
// A batch-1 decode matvec streams every weight once (BebeLM：纯Rust实现的端侧
// 大模型推理引擎, §性能表现: decode is bound by memory bandwidth).  On B200 the
// SMs must also decode ~10^13 weights per second to keep up with HBM, which
// leaves about six issue slots per weight at full issue rate; the decode
// itself takes three (Q8_0), so everything around it has to be nearly free.
// This kernel is built for that:
//   * each CTA owns one contiguous range of rows; its producer warp (one
//     elected lane) moves T whole rows at a time -- one contiguous 1-D bulk
//     async copy of T x row_bytes -- into a ring of S shared-memory stages,
//     completing on the stage's "full" mbarrier, and refills a stage once all
//     consumer warps have arrived on its "empty" mbarrier;
//   * consumer warp w takes R rows of every stage (of its K-segment when rows
//     are longer than 2048 columns): wait, decode, release, reduce -- no
//     copies, cursors or 64-bit bookkeeping in the consumer loop;
//   * lane l's x values for its 64 columns of the K-segment sit in registers
//     for the whole kernel (staged once per CTA through shared memory);
//   * a multi-row butterfly reduces the warp's R partial sums; rows split over
//     K-segments add their warps' partials in shared memory in a fixed order
//     (deterministic, no atomics);
//   * one CTA of 13 warps per SM (at most four warps per SM sub-partition, so
//     128 registers a thread: x and R rows of decode stay in registers) with a
//     ring of ~200 KB; with programmatic dependent launch the next matvec's
//     CTA takes the SM as soon as this one's CTA exits and streams its first
//     stages while the rest of this kernel finishes.
// Every wait is bounded (about a second): a timeout records QMV_DEVERR_TIMEOUT,
// the warp stops decoding but keeps releasing stages, and the producer drains
// its copies before the CTA exits (QMV_DEVERR_DRAIN if that wait runs out too).
#pragma once

#include "qmv_rw.cuh"

namespace qmv {

constexpr int SK_NC = 12;                     // consumer warps
constexpr int SK_THREADS = (SK_NC + 1) * 32;  // + one producer warp
constexpr int SK_MAX_STAGES = 8;
constexpr int SK_SEG = 2048;                  // columns of one K-segment: 64 per lane
constexpr int SK_MAX_KSEGS = 4;               // rows up to 8192 columns (ksegs divides SK_NC)
constexpr int SK_HDR = 256;                   // mbarriers: full[8], empty[8], x_done
constexpr int SK_PART = 2 * SK_NC * 4 * 4;    // K-segment partials (SK_NC * R <= 48 floats), double-buffered

struct SkParams {
    const uint8_t *W;
    const float *x;          // [cols]
    float *y;                // [rows]
    int64_t rows;
    int64_t row_bytes;
    int64_t units_q;         // CTA c owns units_q + (c < units_r) units of `gran` rows
    int32_t units_r;
    int32_t gran;            // rows per unit: gran * row_bytes is a multiple of 16 bytes
    int32_t cols;
    int32_t ksegs;           // consumer warps per row (1, 2 or 4)
    int32_t seg_bytes;       // bytes of one 2048-column K-segment of a row
    int32_t tile_rows;       // T = (SK_NC / ksegs) * R rows per stage
    int32_t n_stage;         // S
    int32_t stage_pitch;     // bytes per stage slot (multiple of 128, >= T * row_bytes + 16)
    int32_t x_in_ring;       // 1: x is staged in ring slot S-1 before its first fill
    int32_t x_off;           // else: byte offset of the x area from the ring start
    int *err;
    uint32_t debug_extra_tx; // test hook: bytes expected per stage beyond those copied (0 in use)
};

// x value layout in registers for one lane's 64-column slice of a K-segment:
// the same slice geometry and pairing as the warp-ring kernel.
template <int FMT>
__device__ __forceinline__ void sk_load_x(uint32_t xs, int seg, int ncols, int lane, float2 (&xr)[16][2],
                                          float &xsa, float &xsb)
{
    rw_load_x_smem<FMT>(xs, seg, ncols, lane, xr, xsa, xsb);
}

template <int FMT, int R>
__global__ void __launch_bounds__(SK_THREADS, 1) qmv_sk_kernel(const __grid_constant__ SkParams p)
{
    static_assert(R == 1 || R == 2 || R == 4, "rows per consumer warp");
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = (int)threadIdx.x >> 5, lane = (int)threadIdx.x & 31;
    const uint32_t sraw = smem_addr(smem);
    const uint32_t sbase = (sraw + 127u) & ~127u;          // the launch adds 128 spare bytes
    const uint32_t full0 = sbase, empty0 = sbase + 8u * SK_MAX_STAGES, xdone = sbase + 16u * SK_MAX_STAGES;
    volatile int *const abort_flag = reinterpret_cast<volatile int *>(smem + (sbase - sraw) + 16 * SK_MAX_STAGES + 8);
    const uint32_t part0 = sbase + (uint32_t)SK_HDR;
    const uint32_t ring = part0 + (uint32_t)SK_PART;
    const int S = p.n_stage;
    const uint32_t pitch = (uint32_t)p.stage_pitch;
    const uint32_t xs = p.x_in_ring ? ring + (uint32_t)(S - 1) * pitch : ring + (uint32_t)p.x_off;

    // this CTA's rows
    const int c = (int)blockIdx.x;
    const int64_t u0 = (int64_t)c * p.units_q + min(c, p.units_r);
    const int64_t r_begin = u0 * p.gran;
    const int64_t r_end = min(p.rows, (u0 + p.units_q + (c < p.units_r ? 1 : 0)) * p.gran);
    const int T = p.tile_rows;
    const int n_st = r_end > r_begin ? (int)((r_end - r_begin + T - 1) / T) : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full0 + 8u * (uint32_t)s, 1);
            mbar_init(empty0 + 8u * (uint32_t)s, SK_NC);
        }
        mbar_init(xdone, SK_NC);
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    pdl_launch_dependents();

    if (warp == SK_NC) {
        // ------------------------------------------------------ producer --
        // Weights do not depend on earlier kernels: no griddepcontrol.wait here.
        if (lane == 0) {
            const uint64_t row_bytes = (uint64_t)p.row_bytes;
            const uint8_t *src = p.W + (uint64_t)r_begin * row_bytes;
            const uint64_t stage_bytes = (uint64_t)T * row_bytes;
            int issued = 0;
            bool ok = true;
            for (int i = 0; i < n_st && ok; ++i) {
                const int slot = i % S;
                const int round = i / S;
                if (round > 0) ok = mbar_wait_bounded(empty0 + 8u * (uint32_t)slot, (uint32_t)((round - 1) & 1));
                else if (p.x_in_ring && slot == S - 1) ok = mbar_wait_bounded(xdone, 0u);
                if (!ok) {
                    atomicOr(p.err, DEVERR_TIMEOUT);
                    break;
                }
                if (*abort_flag) break;           // a consumer timed out: stop re-arming stages
                const int64_t r0 = r_begin + (int64_t)i * T;
                const uint32_t bytes = (uint32_t)(min((int64_t)T, r_end - r0) * p.row_bytes);
                const uint32_t full = full0 + 8u * (uint32_t)slot;
                // the slot was last read (and x, in slot S-1, written) through the generic proxy
                if (round > 0 || (p.x_in_ring && slot == S - 1)) fence_proxy_async_smem();
                mbar_arrive_expect_tx(full, bytes + p.debug_extra_tx);
                bulk_g2s(ring + (uint32_t)slot * pitch, src, bytes, full);
                src += stage_bytes;
                ++issued;
            }
            // let every copy land before the CTA can exit
            for (int i = max(0, issued - S); i < issued; ++i) {
                if (!mbar_wait_bounded(full0 + 8u * (uint32_t)(i % S), (uint32_t)((i / S) & 1))) {
                    atomicOr(p.err, DEVERR_DRAIN);
                    break;
                }
            }
        }
        return;
    }

    // -------------------------------------------------------- consumers --
    pdl_wait();                                    // x is the previous kernel's output
    {
        const float4 *src = reinterpret_cast<const float4 *>(p.x);
        for (int f = (int)threadIdx.x; f < (p.cols >> 2); f += SK_NC * 32)
            sts_f4(xs + 16u * rw_xswz((uint32_t)f), __ldg(src + f));
    }
    named_bar_sync(1, SK_NC * 32);
    const int ks = warp % p.ksegs, rs = warp / p.ksegs;
    const int seg_cols = min(SK_SEG, p.cols - ks * SK_SEG);
    float2 xr[16][2];
    float xsa = 0.f, xsb = 0.f;
    sk_load_x<FMT>(xs, ks, seg_cols, lane, xr, xsa, xsb);
    __syncwarp();
    if (lane == 0) mbar_arrive(xdone);             // the x area may now become ring slot S-1

    const bool have = 64 * (lane + 1) <= seg_cols;
    const Q4kSel sel = q4k_sel(lane & 3);
    const uint32_t row_bytes = (uint32_t)p.row_bytes;
    // this lane's slice within a row of a stage
    uint32_t slice = (uint32_t)ks * (uint32_t)p.seg_bytes;
    if (FMT == FMT_Q8_0) slice += 68u * (uint32_t)lane;
    else if (FMT == FMT_Q4_K) slice += 144u * (uint32_t)(lane >> 2);
    else slice += 210u * (uint32_t)(lane >> 2);
    const int q6h = (lane >> 1) & 1, q6l = 16 * (lane & 1);
    constexpr int SH = 5 - Log2<R>::v;
    const bool leader = (lane & ((1 << SH) - 1)) == 0;
    const int kl = lane >> SH;                     // row (of the warp's R) a leader holds after the butterfly
    auto xp = [&](int gq, float2 &x02, float2 &x13) {
        x02 = xr[gq][0];
        x13 = xr[gq][1];
    };

    bool dead = false;
    for (int i = 0; i < n_st; ++i) {
        const int slot = i % S;
        const uint32_t st = ring + (uint32_t)slot * pitch;
        if (!dead && !__all_sync(0xFFFFFFFFu, mbar_wait_bounded(full0 + 8u * (uint32_t)slot, (uint32_t)((i / S) & 1)))) {
            if (lane == 0) {
                atomicOr(p.err, DEVERR_TIMEOUT);
                *abort_flag = 1;
            }
            dead = true;                          // no more waits; stages are still released
        }
        const int64_t r0 = r_begin + (int64_t)i * T;
        const int tr = (int)min((int64_t)T, r_end - r0);
        float acc[R];
#pragma unroll
        for (int k = 0; k < R; ++k) {
            acc[k] = 0.f;
            const int rl = rs * R + k;
            if (!dead && have && rl < tr) {
                const uint32_t a = st + (uint32_t)rl * row_bytes + slice;
                if (FMT == FMT_Q8_0) acc[k] = q8_0_dot_pair(a, xp);
                else if (FMT == FMT_Q4_K) acc[k] = q4_k_dot1<false>(a, lane & 3, sel, xp, xsa, xsb);
                else acc[k] = q6_k_dot1(a, q6h, q6l, xp);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8u * (uint32_t)slot);   // the stage may be refilled
        warp_transpose_reduce<R>(acc, lane);
        const int rl = rs * R + kl;
        if (p.ksegs == 1) {
            if (leader && rl < tr) p.y[r0 + rl] = acc[0];
        } else {
            // partials of the row's K-segments, added in K order by the first one
            const uint32_t pb = part0 + (uint32_t)(i & 1) * (uint32_t)(SK_PART / 2);
            if (leader) sts_f32(pb + 4u * (uint32_t)(rl * p.ksegs + ks), acc[0]);
            named_bar_sync(2 + rs, 32 * p.ksegs);
            if (ks == 0 && leader && rl < tr) {
                float v = 0.f;
                for (int k2 = 0; k2 < p.ksegs; ++k2) v += lds_f32(pb + 4u * (uint32_t)(rl * p.ksegs + k2));
                p.y[r0 + rl] = v;
            }
        }
    }
}

// Defined per format in qmv_fmt_*.cu.
template <int FMT>
cudaError_t launch_sk(const SkParams &p, int R, dim3 grid, size_t smem, cudaStream_t stream, bool pdl);

}  // namespace qmv
