// qmv_sk.cuh -- the one-token streaming matvec: one producer warp, twelve
// consumer warps, multi-row stages.
//
// A batch-1 decode matvec streams every weight once (BebeLM：纯Rust实现的端侧
// 大模型推理引擎, §性能表现: decode is bound by memory bandwidth).  On B200 the
// SMs must also decode ~10^13 weights per second to keep up with HBM, which
// leaves about six issue slots per weight at full issue rate; the decode
// itself takes three (Q8_0), so everything around it has to be nearly free.
// This kernel is built for that:
//   * each CTA owns one contiguous range of output rows; its producer warp
//     (one elected lane) fills a ring of S shared-memory stages.  A stage
//     holds T rows, contiguous per matrix, filled by a few 1-D bulk async
//     copies of whole rows (one per matrix and run of rows of one expert)
//     that complete on the stage's "full" mbarrier; the producer issues the
//     first stages of a plain matrix before the CTA-wide barrier, and tags
//     the copies to leave L2 first.  A stage is refilled once all twelve
//     consumer warps have arrived on its "empty" mbarrier;
//   * consumer warp w = (row slot, K-segment) takes its R rows of every stage
//     (its 2048-column K-segment when rows are longer): wait, decode, release,
//     reduce -- no copies, cursors or 64-bit bookkeeping in the consumer loop;
//   * lane l's x values for its 64 columns of the K-segment sit in registers
//     for the whole kernel (staged once per CTA through shared memory);
//   * a multi-row butterfly reduces the warp's partial sums; rows split over
//     K-segments add their warps' partials in shared memory in a fixed order
//     (deterministic, no atomics);
//   * one CTA of 13 warps per SM (at most four warps per SM sub-partition, so
//     128 registers a thread) with a ring of up to ~200 KB; with programmatic
//     dependent launch the next kernel's CTA takes the SM as soon as this
//     one's CTA exits and streams its first stages while the rest finishes.
// Three forms share the body (BebeLM page, §核心算子, MoE前馈网络):
//   SK_PLAIN   y = W x (a matrix, or a row-concatenated fused projection);
//   SK_SWIGLU  h[k][r] = silu(G_{ids[k]} x)[r] * (U_{ids[k]} x)[r]: a stage
//              holds T gate rows, then the same T up rows;
//   SK_GATHER  y[r] = sum_k g[k] (D_{ids[k]} h_k)[r]: K-segment k of a row is
//              row r of expert ids[k]'s matrix (a stage holds T rows of each
//              routed expert in turn), weighted and summed in k order.
// An expert id outside [0, n_expert) copies nothing, contributes zero and
// records QMV_DEVERR_EXPERT_ID.  Every wait is bounded (about a second): a
// timeout records QMV_DEVERR_TIMEOUT, the warp stops decoding but keeps
// releasing stages, and the producer drains its copies before the CTA exits
// (QMV_DEVERR_DRAIN if that wait runs out too).
#pragma once

#include "qmv_rw.cuh"

namespace qmv {

constexpr int SK_NC = 12;                     // consumer warps
constexpr int SK_THREADS = (SK_NC + 1) * 32;  // + one producer warp
constexpr int SK_MAX_STAGES = 8;
constexpr int SK_SEG = 2048;                  // columns of one K-segment: 64 per lane
constexpr int SK_MAX_KSEGS = SK_NC;           // K-segments per row: a divisor of SK_NC
constexpr int SK_MAX_RS = SK_NC;              // row slots per stage
// header: full[stage][row slot], empty[stage], x_done, abort flag, segment weights
// (the fused MoE kernel keeps its routed ids and weights, 64 bytes, in front
// of the segment weights)
constexpr int SK_FULL_OFF = 0;
constexpr int SK_EMPTY_OFF = 8 * SK_MAX_STAGES * SK_MAX_RS;           // 768 for 12 consumer warps
constexpr int SK_XDONE_OFF = SK_EMPTY_OFF + 8 * SK_MAX_STAGES;
constexpr int SK_ABORT_OFF = SK_XDONE_OFF + 8;
constexpr int SK_WSEG_OFF = (SK_ABORT_OFF + 8 + 63) / 64 * 64;       // [64 B of MoE routing] float[SK_MAX_KSEGS]
constexpr int SK_HDR = (SK_WSEG_OFF + 64 + 4 * SK_MAX_KSEGS + 127) / 128 * 128;
constexpr int SK_PART = 2 * SK_NC * 4 * 2 * 4;   // partials [row][group][segment] <= NC*R*G floats, double-buffered

enum { SK_PLAIN = 0, SK_SWIGLU = 1, SK_GATHER = 2 };

// 1: the rows (and gate / up groups) of a row slot are decoded by one copy of
// the decode body in a loop, keeping the kernels' code small (a kernel that
// runs a few stages per launch spends much of its time fetching cold
// instructions); 0: fully unrolled.
#ifndef QMV_SK_ROW_LOOP
#define QMV_SK_ROW_LOOP 0
#endif
#if QMV_SK_ROW_LOOP
#define QMV_SK_ROWS_PRAGMA _Pragma("unroll 1")
#else
#define QMV_SK_ROWS_PRAGMA _Pragma("unroll")
#endif

struct SkParams {
    const uint8_t *W;        // PLAIN: the matrix; SWIGLU: gate matrices; GATHER: down matrices
    const uint8_t *W2;       // SWIGLU: up matrices
    int64_t expert_stride;   // SWIGLU / GATHER: bytes from one expert's matrix to the next
    const int32_t *ids;      // SWIGLU / GATHER: routed expert ids [n_sel] (device)
    const float *gw;         // GATHER: expert weights [n_sel] (device)
    int32_t n_expert;
    int32_t n_sel;
    int32_t inter;           // SWIGLU: rows per expert (output row v = k * inter + r)
    int32_t cols;            // columns of one matrix row (GATHER: of one expert's row = one K-segment)
    const float *x;          // PLAIN / SWIGLU: x [cols]; GATHER: h [n_sel][cols]
    float *y;                // [rows]
    int64_t rows;            // output rows (SWIGLU: n_sel * inter)
    int64_t row_bytes;       // bytes of one matrix row (GATHER: of one expert's row)
    int64_t units_q;         // CTA c owns units_q + (c < units_r) units of `gran` rows
    int32_t units_r;
    int32_t gran;            // rows per unit: a multiple of R
    int32_t ksegs;           // consumer warps per row (a divisor of SK_NC)
    int32_t seg_bytes;       // PLAIN / SWIGLU: bytes of one 2048-column K-segment of a row
    int32_t tile_rows;       // T = (SK_NC / ksegs) * R rows per stage
    int32_t n_stage;         // S
    int32_t stage_pitch;     // bytes per stage slot (multiple of 128, >= a stage + 16)
    int32_t x_in_ring;       // 1: x is staged in ring slot S-1 before its first fill
    int32_t x_off;           // else: byte offset of the x area from the ring start
    int32_t x_row;           // several tokens: bytes from one token's staged x row to the next
    // PLAIN with a single K-segment: greedy argmax of y fused into the epilogue
    // (amax_idx != NULL).  Every CTA folds its best (value, row) into *amax_key;
    // the last CTA to arrive on *amax_done writes *amax_idx and puts both back
    // to zero.
    unsigned long long *amax_key;
    unsigned *amax_done;
    int32_t *amax_idx;
    // weights of the next matvec in stream order (NULL: none): once its last
    // copy is issued, CTA c starts moving its share of them into L2, so the
    // next launch finds them there and HBM stays busy across the boundary
    const uint8_t *pf;
    int64_t pf_bytes;
    int *err;
    uint32_t debug_extra_tx; // test hook: bytes expected per row slot beyond those copied (0 in use)
};

__device__ __forceinline__ bool sk_valid(const SkParams &p, int k)
{
    const int e = p.ids[k];
    return e >= 0 && e < p.n_expert;
}

// Starts moving `bytes` (a multiple of 16, 16-byte aligned) of global memory
// into L2 without waiting.  Used on x before griddepcontrol.wait: if the
// previous kernel writes x afterwards, L2 holds its writes all the same.
__device__ __forceinline__ void prefetch_l2(const void *src, uint32_t bytes)
{
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" :: "l"(src), "r"(bytes) : "memory");
}

constexpr int SK_X_MAX_BYTES = 96 * 1024;    // largest x staged in shared memory (24576 floats)
constexpr uint32_t SK_PF_PIECE = 64 * 1024;  // bytes per L2 prefetch request
// Stages of a plain matrix issued before x is loaded (measured on B200: two
// beat one, three and the whole ring -- the Q8_0 gate/up 16384x2048 matvec
// 9.0 against 9.7 us with three of a four-stage ring or the whole ring).
constexpr int SK_HEAD_START = 2;

// Copies x into the swizzled x area of shared memory (float4 d at
// 16 * rw_xswz(d)): n_rows rows of nr float4, row k from src + k * src_row
// floats to float4 k * 512 of the area (SK_SEG columns per row).  A thread
// issues up to eight loads before its first store, so staging up to 12288
// floats costs one memory round trip (the loads queue behind the weight
// copies in flight).
// COHERENT: read through L2 only (x may have been written earlier in the same
// launch by another SM).
template <bool COHERENT>
__device__ __forceinline__ void sk_stage_x(uint32_t xs, const float *src, int n_rows, int nr, int64_t src_row)
{
    constexpr int B = 8;                          // loads in flight per thread and pass
    const int n = n_rows == 1 ? nr : n_rows * (SK_SEG / 4);
#pragma unroll 1
    for (int base = 0; base < n; base += B * SK_NC * 32) {
        float4 v[B];
#pragma unroll
        for (int j = 0; j < B; ++j) {
            const int d = base + (int)threadIdx.x + j * SK_NC * 32;
            const int k = n_rows == 1 ? 0 : d >> 9, c = n_rows == 1 ? d : d & 511;
            if (d < n && c < nr) {
                const float4 *a = reinterpret_cast<const float4 *>(src + (int64_t)k * src_row) + c;
                v[j] = COHERENT ? __ldcg(a) : __ldg(a);
            }
        }
#pragma unroll
        for (int j = 0; j < B; ++j) {
            const int d = base + (int)threadIdx.x + j * SK_NC * 32;
            const int c = n_rows == 1 ? d : d & 511;
            if (d < n && c < nr) sts_f4(xs + 16u * rw_xswz((uint32_t)d), v[j]);
        }
    }
}

template <int FMT, int R, int MODE>
__global__ void __launch_bounds__(SK_THREADS, 1) qmv_sk_kernel(const __grid_constant__ SkParams p)
{
    static_assert(R == 1 || R == 2 || R == 4, "rows per consumer warp");
    constexpr int G = MODE == SK_SWIGLU ? 2 : 1;      // matrices per row slot (gate and up)
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = (int)threadIdx.x >> 5, lane = (int)threadIdx.x & 31;
    const uint32_t sraw = smem_addr(smem);
    const uint32_t sbase = (sraw + 127u) & ~127u;          // the launch adds 128 spare bytes
    uint8_t *const sgen = smem + (sbase - sraw);
    const uint32_t full0 = sbase + SK_FULL_OFF, empty0 = sbase + SK_EMPTY_OFF, xdone = sbase + SK_XDONE_OFF;
    volatile int *const abort_flag = reinterpret_cast<volatile int *>(sgen + SK_ABORT_OFF);
    float *const wseg = reinterpret_cast<float *>(sgen + SK_WSEG_OFF);
    const uint32_t part0 = sbase + (uint32_t)SK_HDR;
    const uint32_t ring = part0 + (uint32_t)SK_PART;
    const int S = p.n_stage;
    const uint32_t pitch = (uint32_t)p.stage_pitch;
    const uint32_t xs = p.x_in_ring ? ring + (uint32_t)(S - 1) * pitch : ring + (uint32_t)p.x_off;
    // one "full" mbarrier per stage: every consumer waits for the whole stage
    auto full_bar = [&](int s) { return full0 + 8u * (uint32_t)s; };

    // this CTA's rows
    const int c = (int)blockIdx.x;
    const int64_t u0 = (int64_t)c * p.units_q + min(c, p.units_r);
    const int64_t r_begin = u0 * p.gran;
    const int64_t r_end = min(p.rows, (u0 + p.units_q + (c < p.units_r ? 1 : 0)) * p.gran);
    const int T = p.tile_rows;
    const int n_st = r_end > r_begin ? (int)((r_end - r_begin + T - 1) / T) : 0;

    const uint64_t rbw = (uint64_t)p.row_bytes;   // bytes of one matrix row
    const int n_xrow = MODE == SK_GATHER ? min(p.n_sel, p.ksegs) : 1;
    // weights are read once per decode step: evict them from L2 first
    const uint64_t wpol = l2_evict_first_policy();
    auto wcopy = [&](uint32_t dst, const uint8_t *src, uint32_t bytes, uint32_t bar) {
        bulk_g2s_hint(dst, src, bytes, bar, wpol);
    };
    // The copies of stage i into ring slot `slot` (producer lane 0), all
    // completing on the slot's one "full" barrier.  A stage's T rows are
    // contiguous in shared memory per matrix: PLAIN one copy; SWIGLU the gate
    // rows then (at T rows) the up rows, one copy of each per run of rows of
    // one expert; GATHER expert k's rows at k T rows, one copy per expert.
    auto issue = [&](int i, int slot) {
        const int64_t r0 = r_begin + (int64_t)i * T;
        const int tr = (int)min((int64_t)T, r_end - r0);
        const uint32_t st = ring + (uint32_t)slot * pitch;
        const uint32_t full = full_bar(slot);
        if (MODE == SK_PLAIN) {
            const uint32_t bytes = (uint32_t)tr * (uint32_t)rbw;
            mbar_arrive_expect_tx(full, bytes + p.debug_extra_tx);
            wcopy(st, p.W + (uint64_t)r0 * rbw, bytes, full);
        } else if (MODE == SK_SWIGLU) {
            // output row v = k * inter + r (expert slot k, row r of its matrices)
            int k = (int)(r0 / p.inter);
            int r = (int)(r0 - (int64_t)k * p.inter);
            uint32_t total = 0;
            for (int done = 0, kk = k, rr = r; done < tr; ++kk, rr = 0) {
                const int run = min(tr - done, p.inter - rr);
                if (sk_valid(p, kk)) total += 2u * (uint32_t)run * (uint32_t)rbw;
                done += run;
            }
            mbar_arrive_expect_tx(full, total + p.debug_extra_tx);
            for (int done = 0; done < tr; ++k, r = 0) {
                const int run = min(tr - done, p.inter - r);
                if (sk_valid(p, k)) {
                    const uint64_t off = (uint64_t)p.ids[k] * (uint64_t)p.expert_stride + (uint64_t)r * rbw;
                    const uint32_t dst = st + (uint32_t)done * (uint32_t)rbw;
                    const uint32_t bytes = (uint32_t)run * (uint32_t)rbw;
                    wcopy(dst, p.W + off, bytes, full);
                    wcopy(dst + (uint32_t)T * (uint32_t)rbw, p.W2 + off, bytes, full);
                }
                done += run;
            }
        } else {
            const int n_seg = min(p.n_sel, p.ksegs);   // a stage holds ksegs experts' rows
            const uint32_t bytes = (uint32_t)tr * (uint32_t)rbw;
            uint32_t total = 0;
            for (int k = 0; k < n_seg; ++k)
                if (sk_valid(p, k)) total += bytes;
            mbar_arrive_expect_tx(full, total + p.debug_extra_tx);
            for (int k = 0; k < n_seg; ++k) {
                if (!sk_valid(p, k)) continue;
                wcopy(st + (uint32_t)(k * T) * (uint32_t)rbw,
                      p.W + (uint64_t)p.ids[k] * (uint64_t)p.expert_stride + (uint64_t)r0 * rbw, bytes, full);
            }
        }
    };

    // The producer initialises the barriers and, for a plain matrix (whose
    // weights depend on no earlier kernel), issues the first SK_HEAD_START
    // stages before the CTA-wide barrier: the copies are in flight from the
    // CTA's start.  The other threads meanwhile start x on its way into L2.
    int pre = 0;
    if (warp == SK_NC && lane == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty0 + 8u * (uint32_t)s, SK_NC);
        }
        mbar_init(xdone, SK_NC);
        *abort_flag = 0;
        fence_mbar_init();
        if (MODE == SK_PLAIN) {
            pre = min(n_st, min(p.x_in_ring ? S - 1 : S, SK_HEAD_START));
            for (int i = 0; i < pre; ++i) issue(i, i);
        }
    } else if (threadIdx.x == 0) {
        prefetch_l2(p.x, (uint32_t)(n_xrow * p.cols * 4));
    }
    __syncthreads();
    pdl_launch_dependents();

    if (warp == SK_NC) {
        // ------------------------------------------------------ producer --
        if (lane != 0) return;
        // routed experts depend on the previous kernel (ids)
        if (MODE != SK_PLAIN) pdl_wait();
        int issued = pre;
        bool ok = true;
        // after the head start, the rest of the ring waits until x is in the
        // warps' registers: x's loads then do not queue behind a whole ring of
        // weight copies (the head start keeps HBM busy meanwhile)
        if (MODE == SK_PLAIN && pre < n_st && !mbar_wait_bounded_block(xdone, 0u)) {
            atomicOr(p.err, DEVERR_TIMEOUT);
            ok = false;
        }
        for (int i = pre; i < n_st && ok; ++i) {
            const int slot = i % S;
            const int round = i / S;
            if (round > 0) ok = mbar_wait_bounded_block(empty0 + 8u * (uint32_t)slot, (uint32_t)((round - 1) & 1));
            else if (p.x_in_ring && slot == S - 1) ok = mbar_wait_bounded_block(xdone, 0u);
            if (!ok) {
                atomicOr(p.err, DEVERR_TIMEOUT);
                break;
            }
            if (*abort_flag) break;           // a consumer timed out: stop re-arming stages
            // the slot was last read (and x, in slot S-1, written) through the generic proxy
            if (round > 0 || (p.x_in_ring && slot == S - 1)) fence_proxy_async_smem();
            issue(i, slot);
            ++issued;
        }
        if (ok && p.pf != nullptr) {
            // this CTA's share of the next matvec's weights (16-byte granules)
            const uint64_t total = (uint64_t)p.pf_bytes & ~15ull;
            const uint64_t share = ((total / gridDim.x) + 15u) & ~15ull;
            const uint64_t b0 = share * blockIdx.x;
            const uint64_t b1 = min(b0 + share, total);
            for (uint64_t o = b0; o < b1; o += SK_PF_PIECE)
                prefetch_l2(p.pf + o, (uint32_t)min((uint64_t)SK_PF_PIECE, b1 - o));
        }
        // let every copy land before the CTA can exit
        bool drained = true;
        for (int i = max(0, issued - S); i < issued && drained; ++i) {
            if (!mbar_wait_bounded_block(full_bar(i % S), (uint32_t)((i / S) & 1))) {
                atomicOr(p.err, DEVERR_DRAIN);
                drained = false;
            }
        }
        return;
    }

    // -------------------------------------------------------- consumers --
    pdl_wait();                                    // x, h, ids and weights come from earlier kernels
    if (MODE == SK_GATHER) {
        // h_k at float offset k * SK_SEG of the x area (a K-segment per expert)
        sk_stage_x<false>(xs, p.x, n_xrow, p.cols >> 2, p.cols);
        if ((int)threadIdx.x < SK_MAX_KSEGS) {
            const int k = (int)threadIdx.x;
            float w = 0.f;
            if (k < p.n_sel) {
                if (sk_valid(p, k)) w = p.gw[k];
                else atomicOr(p.err, DEVERR_EXPERT_ID);
            }
            wseg[k] = w;
        }
    } else {
        sk_stage_x<false>(xs, p.x, 1, p.cols >> 2, 0);
        if (MODE == SK_SWIGLU && (int)threadIdx.x < p.n_sel && !sk_valid(p, (int)threadIdx.x))
            atomicOr(p.err, DEVERR_EXPERT_ID);
    }
    named_bar_sync(1, SK_NC * 32);
    const int ks = warp % p.ksegs, rs = warp / p.ksegs;
    int seg_cols;
    if (MODE == SK_GATHER) seg_cols = ks < p.n_sel && sk_valid(p, ks) ? p.cols : 0;
    else seg_cols = min(SK_SEG, p.cols - ks * SK_SEG);
    float2 xr[16][2];
    float xsa = 0.f, xsb = 0.f;
    rw_load_x_smem<FMT>(xs, ks, seg_cols, lane, xr, xsa, xsb);
    __syncwarp();
    if (lane == 0) mbar_arrive(xdone);             // the x area may now become ring slot S-1

    const bool have = 64 * (lane + 1) <= seg_cols;
    const Q4kSel sel = q4k_sel(lane & 3);
    const uint32_t rb = (uint32_t)p.row_bytes;
    // this lane's slice of the warp's first row in a stage (layout: issue());
    // SWIGLU's up rows follow the gate rows at gst
    uint32_t slice = (uint32_t)(rs * R) * rb;
    slice += (uint32_t)ks * (MODE == SK_GATHER ? (uint32_t)T * rb : (uint32_t)p.seg_bytes);
    slice += lane_slice_off<FMT>(lane);
    const uint32_t gst = (uint32_t)T * rb;
    constexpr int V = G * R;
    constexpr int SH = 5 - Log2<V>::v;
    const bool leader = (lane & ((1 << SH) - 1)) == 0;
    const int vi = lane >> SH;                     // value (group * R + row) a leader holds after the butterfly
    const int vg = vi / R, vk = vi % R;
    auto xp = [&](int gq, float2 &x02, float2 &x13) {
        x02 = xr[gq][0];
        x13 = xr[gq][1];
    };

    bool dead = false;
    int slot = 0;
    uint32_t phase = 0, st = ring;
    int64_t r0 = r_begin;
    float best_v = 0.f;                            // fused argmax: this lane's candidate
    int best_i = -1;
    for (int i = 0; i < n_st; ++i) {
        const int ra = min(R, (int)min((int64_t)T, r_end - r0) - rs * R);     // rows of this row slot
        bool rowok = ra > 0;
        if (MODE == SK_SWIGLU && rowok) rowok = sk_valid(p, (int)(r0 + rs * R) / p.inter);
        if (ra > 0 && !dead && !__all_sync(0xFFFFFFFFu, mbar_wait_bounded_block(full_bar(slot), phase))) {
            if (lane == 0) {
                atomicOr(p.err, DEVERR_TIMEOUT);
                *abort_flag = 1;
            }
            dead = true;                          // no more waits; stages are still released
        }
        float acc[V];
#pragma unroll
        for (int j = 0; j < V; ++j) acc[j] = 0.f;
        QMV_SK_ROWS_PRAGMA
        for (int j = 0; j < V; ++j) {                // j = g * R + k
            const int k = j % R;
            float d = 0.f;
            if (!dead && rowok && have && k < ra) {
                const uint32_t a = st + slice + (uint32_t)(j / R) * gst + (uint32_t)k * rb;
                d = lane_dot<FMT>(a, lane, sel, xp, xsa, xsb);
            }
#pragma unroll
            for (int j2 = 0; j2 < V; ++j2)
                if (j2 == j) acc[j2] = d;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8u * (uint32_t)slot);   // the stage may be refilled
        warp_transpose_reduce<V>(acc, lane);
        const int64_t row = r0 + rs * R + vk;
        if (p.ksegs == 1) {
            if (MODE == SK_SWIGLU) {
                const float u = __shfl_down_sync(0xFFFFFFFFu, acc[0], R << SH);    // the up value of row vk
                if (leader && vg == 0 && vk < ra) p.y[row] = rowok ? acc[0] / (1.0f + expf(-acc[0])) * u : 0.f;
            } else if (leader && vk < ra) {
                const float v = MODE == SK_GATHER ? wseg[0] * acc[0] : acc[0];
                p.y[row] = v;
                if (MODE == SK_PLAIN && v == v) argmax_merge(best_v, best_i, v, (int)row);
            }
        } else {
            // partials of the row's K-segments, added in K order by segment 0
            const uint32_t pb = part0 + (uint32_t)(i & 1) * (uint32_t)(SK_PART / 2);
            const int nk = p.ksegs;
            if (leader) sts_f32(pb + 4u * (uint32_t)(((rs * R + vk) * G + vg) * nk + ks), acc[0]);
            named_bar_sync(2 + rs, 32 * nk);
            if (ks == 0 && leader && vg == 0 && vk < ra) {
                float s0 = 0.f, s1 = 0.f;
                const uint32_t e0 = pb + 4u * (uint32_t)((rs * R + vk) * G * nk);
                for (int k2 = 0; k2 < nk; ++k2) {
                    const float v = lds_f32(e0 + 4u * (uint32_t)k2);
                    if (MODE == SK_GATHER) s0 = fmaf(wseg[k2], v, s0);
                    else s0 += v;
                    if (MODE == SK_SWIGLU) s1 += lds_f32(e0 + 4u * (uint32_t)(nk + k2));
                }
                p.y[row] = MODE == SK_SWIGLU ? (rowok ? s0 / (1.0f + expf(-s0)) * s1 : 0.f) : s0;
            }
        }
        if (++slot == S) {
            slot = 0;
            phase ^= 1u;
        }
        st = ring + (uint32_t)slot * pitch;
        r0 += T;
    }
    if (MODE == SK_PLAIN && p.amax_idx != nullptr) {
        // CTA's best candidate (warp butterfly, then warp 0 over the warps'
        // results in the partials area), one atomic per CTA
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1)
            argmax_merge(best_v, best_i, __shfl_xor_sync(0xFFFFFFFFu, best_v, o), __shfl_xor_sync(0xFFFFFFFFu, best_i, o));
        named_bar_sync(1, SK_NC * 32);            // every warp is past its last partials
        if (lane == 0) {
            sts_f32(part0 + 8u * (uint32_t)warp, best_v);
            sts_f32(part0 + 8u * (uint32_t)warp + 4u, __int_as_float(best_i));
        }
        named_bar_sync(1, SK_NC * 32);
        if (warp == 0) {
            float v = 0.f;
            int bi = -1;
            if (lane < SK_NC) {
                v = lds_f32(part0 + 8u * (uint32_t)lane);
                bi = __float_as_int(lds_f32(part0 + 8u * (uint32_t)lane + 4u));
            }
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1)
                argmax_merge(v, bi, __shfl_xor_sync(0xFFFFFFFFu, v, o), __shfl_xor_sync(0xFFFFFFFFu, bi, o));
            if (lane == 0) {
                if (bi >= 0) atomicMax(p.amax_key, argmax_key(v, bi));
                __threadfence();
                if (atomicAdd(p.amax_done, 1u) == gridDim.x - 1u) {     // the last CTA
                    __threadfence();
                    const unsigned long long k = atomicExch(p.amax_key, 0ull);
                    atomicExch(p.amax_done, 0u);
                    *p.amax_idx = k ? (int32_t)(0xFFFFFFFFu - (uint32_t)(k & 0xFFFFFFFFull)) : -1;
                }
            }
        }
    }
}

// Defined per format in qmv_fmt_*.cu.
template <int FMT>
cudaError_t launch_sk(const SkParams &p, int mode, int R, dim3 grid, size_t smem, cudaStream_t stream, bool pdl);

// ---------------------------------------------------------------------------
// The whole MoE FFN step in one cooperative launch (BebeLM page, §核心算子,
// MoE前馈网络: sigmoid router, top-k by the biased score, weights normalised
// over the unbiased scores; SwiGLU experts):
//   1. every CTA routes on its own (the same f32 arithmetic as moe_route, so
//      the same ids and weights) or reads given ids / weights; CTA 0 writes
//      them out;
//   2. h_k = silu(G_{ids[k]} x) * (U_{ids[k]} x) over this CTA's share of the
//      n_sel * inter rows (the SK_SWIGLU form), stored to h;
//   3. a grid barrier (h complete), then y = sum_k g_k D_{ids[k]} h_k over this
//      CTA's share of the hidden rows (the SK_GATHER form).
// The producer streams the stages of step 2 and then of step 3 without
// waiting for the grid, so the routed down weights are already in shared
// memory when the consumers cross the barrier.
constexpr int SKM_MAX_EXPERTS = 256;          // routed on the device: eight per lane

struct SkMoeParams {
    const float *logits;     // [n_expert]: route on the device; NULL: ids / gw given
    const float *bias;       // [n_expert]
    int32_t *ids_out;        // routed: [n_sel] written by CTA 0 (or NULL)
    float *g_out;            // routed: [n_sel] (or NULL)
    const int32_t *ids;      // given ids [n_sel] (logits == NULL)
    const float *gw;         // given weights [n_sel]
    int32_t n_expert;
    int32_t n_sel;
    const uint8_t *G, *U;    // gate / up experts: [inter x hidden] each
    int64_t gu_stride;
    int64_t gu_row_bytes;
    const uint8_t *D;        // down experts: [hidden x inter]
    int64_t d_stride;
    int64_t d_row_bytes;
    int32_t hidden, inter;
    const float *x;          // [hidden]
    float *h;                // [n_sel][inter]
    float *y;                // [hidden]
    // step 2 (gate/up): K-segments of hidden, rows per stage, CTA split
    int32_t a_ksegs, a_seg_bytes, a_T;
    int64_t a_units_q;
    int32_t a_units_r;
    // step 3 (down): one K-segment per routed expert
    int32_t b_ksegs, b_T;
    int64_t b_units_q;
    int32_t b_units_r;
    int32_t n_stage, stage_pitch, x_off;
    unsigned *sync;          // {arrivals, exits} of the grid barrier (caller workspace), zero between launches
    int *err;
    uint32_t debug_extra_tx;
};

// Top-k routing by one warp, n_expert <= SKM_MAX_EXPERTS: the arithmetic and
// tie rule of moe_route_kernel (sigmoid score s, biased b = s + bias, k rounds
// of a warp argmax over b with ties to the lower index, g = s / sum of the
// chosen s in k order).  Results in sids / sg (shared memory).
__device__ __forceinline__ void skm_route(const float *logits, const float *bias, int n_expert, int top_k, int lane,
                                          int *sids, float *sg)
{
    float sc[SKM_MAX_EXPERTS / 32], bb[SKM_MAX_EXPERTS / 32];
    unsigned taken = 0;
#pragma unroll
    for (int j = 0; j < SKM_MAX_EXPERTS / 32; ++j) {
        const int e = lane + 32 * j;
        sc[j] = 0.f;
        bb[j] = 0.f;
        if (e < n_expert) {
            const float s = 1.0f / (1.0f + expf(-logits[e]));
            sc[j] = s;
            bb[j] = s + bias[e];
        }
    }
    float total = 0.f;
    for (int k = 0; k < top_k; ++k) {
        float bv = 0.f, sv = 0.f;
        int bi = -1;
#pragma unroll
        for (int j = 0; j < SKM_MAX_EXPERTS / 32; ++j) {
            const int e = lane + 32 * j;
            if (e < n_expert && !((taken >> j) & 1u) && (bi < 0 || bb[j] > bv)) {
                bv = bb[j];
                bi = e;
                sv = sc[j];
            }
        }
        for (int o = 16; o >= 1; o >>= 1) {
            const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, o);
            const int oi = __shfl_xor_sync(0xFFFFFFFFu, bi, o);
            const float os = __shfl_xor_sync(0xFFFFFFFFu, sv, o);
            if ((oi >= 0) && (bi < 0 || ov > bv || (ov == bv && oi < bi))) {
                bv = ov;
                bi = oi;
                sv = os;
            }
        }
        if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
        if (lane == 0) {
            sids[k] = bi;
            sg[k] = sv;
        }
        total += sv;
    }
    __syncwarp();
    if (lane < top_k) sg[lane] = sg[lane] / total;
    __syncwarp();
}

template <int FMT, int R>
__global__ void __launch_bounds__(SK_THREADS, 1) qmv_skm_kernel(const __grid_constant__ SkMoeParams p)
{
    static_assert(R == 1 || R == 2, "rows per consumer warp");
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = (int)threadIdx.x >> 5, lane = (int)threadIdx.x & 31;
    const uint32_t sraw = smem_addr(smem);
    const uint32_t sbase = (sraw + 127u) & ~127u;          // the launch adds 128 spare bytes
    uint8_t *const sgen = smem + (sbase - sraw);
    const uint32_t full0 = sbase + SK_FULL_OFF, empty0 = sbase + SK_EMPTY_OFF;
    volatile int *const abort_flag = reinterpret_cast<volatile int *>(sgen + SK_ABORT_OFF);
    int *const sids = reinterpret_cast<int *>(sgen + SK_WSEG_OFF);              // [8]
    float *const sg = reinterpret_cast<float *>(sgen + SK_WSEG_OFF + 32);      // [8] routed weights
    float *const wseg = reinterpret_cast<float *>(sgen + SK_WSEG_OFF + 64);    // [ksegs] segment weights (0: invalid)
    const uint32_t part0 = sbase + (uint32_t)SK_HDR;
    const uint32_t ring = part0 + (uint32_t)SK_PART;
    const uint32_t xs = ring + (uint32_t)p.x_off;
    const int S = p.n_stage;
    const uint32_t pitch = (uint32_t)p.stage_pitch;
    const int c = (int)blockIdx.x;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full0 + 8u * (uint32_t)s, 1);
            mbar_init(empty0 + 8u * (uint32_t)s, SK_NC);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    // this CTA's rows of step 2 (gate/up: n_sel * inter) and step 3 (down: hidden)
    const int64_t a_u0 = (int64_t)c * p.a_units_q + min(c, p.a_units_r);
    const int64_t a_begin = a_u0 * R;
    const int64_t a_end = min((int64_t)p.n_sel * p.inter, (a_u0 + p.a_units_q + (c < p.a_units_r ? 1 : 0)) * R);
    const int64_t b_u0 = (int64_t)c * p.b_units_q + min(c, p.b_units_r);
    const int64_t b_begin = b_u0 * R;
    const int64_t b_end = min((int64_t)p.hidden, (b_u0 + p.b_units_q + (c < p.b_units_r ? 1 : 0)) * R);
    const int na = a_end > a_begin ? (int)((a_end - a_begin + p.a_T - 1) / p.a_T) : 0;
    const int nb = b_end > b_begin ? (int)((b_end - b_begin + p.b_T - 1) / p.b_T) : 0;
    // The producer's parameters, read while warp 0 routes and kept opaque so
    // that they are not read again from the parameter bank after the barrier:
    // a constant-cache miss there would sit between the routing and the first
    // weight copy.
    int n_expert = p.n_expert;
    const uint8_t *pG = nullptr, *pU = nullptr, *pD = nullptr;
    uint64_t gus = 0, dstr = 0, rga = 0, rgb = 0;
    int aT = 0, bT = 0, inter = 0, nsel = 0, bks = 0;
    uint32_t xtx = 0;
    if (warp == SK_NC && lane == 0) {
        pG = p.G; pU = p.U; pD = p.D;
        gus = (uint64_t)p.gu_stride; dstr = (uint64_t)p.d_stride;
        rga = (uint64_t)p.gu_row_bytes; rgb = (uint64_t)p.d_row_bytes;
        aT = p.a_T; bT = p.b_T; inter = p.inter; nsel = p.n_sel; bks = p.b_ksegs; xtx = p.debug_extra_tx;
        asm volatile("" : "+l"(pG), "+l"(pU), "+l"(pD), "+l"(gus), "+l"(dstr), "+l"(rga), "+l"(rgb));
        asm volatile("" : "+r"(aT), "+r"(bT), "+r"(inter), "+r"(nsel), "+r"(bks), "+r"(xtx), "+r"(n_expert));
    }
    if (warp == 0) {
        if (p.logits) {
            skm_route(p.logits, p.bias, p.n_expert, p.n_sel, lane, sids, sg);
            if (c == 0 && lane < p.n_sel) {
                if (p.ids_out) p.ids_out[lane] = sids[lane];
                if (p.g_out) p.g_out[lane] = sg[lane];
            }
        } else if (lane < p.n_sel) {
            sids[lane] = p.ids[lane];
            sg[lane] = p.gw[lane];
        }
        __syncwarp();
        if (lane < SK_MAX_KSEGS) {
            const bool v = lane < p.n_sel && sids[lane] >= 0 && sids[lane] < p.n_expert;
            wseg[lane] = v ? sg[lane] : 0.f;
            if (lane < p.n_sel && !v && c == 0) atomicOr(p.err, DEVERR_EXPERT_ID);
        }
    }
    __syncthreads();
    auto valid = [&](int k) { return sids[k] >= 0 && sids[k] < n_expert; };

    if (warp == SK_NC) {
        // ------------------------------------------------------ producer --
        if (lane != 0) return;
        bool ok = true;
        int i = 0;
        for (; i < na + nb && ok; ++i) {
            const int slot = i % S, round = i / S;
            if (round > 0 && !mbar_wait_bounded_block(empty0 + 8u * (uint32_t)slot, (uint32_t)((round - 1) & 1))) {
                atomicOr(p.err, DEVERR_TIMEOUT);
                ok = false;
                break;
            }
            if (*abort_flag) {
                ok = false;
                break;
            }
            if (round > 0) fence_proxy_async_smem();
            const uint32_t st = ring + (uint32_t)slot * pitch;
            const uint32_t full = full0 + 8u * (uint32_t)slot;
            if (i < na) {
                // step 2: the stage's a_T gate rows, then the same up rows (at
                // a_T rows), one copy of each per run of rows of one expert
                const int r0 = (int)(a_begin + (int64_t)i * aT);
                const int tr = min(aT, (int)(a_end - r0));
                const int k0 = r0 / inter, q0 = r0 - k0 * inter;
                uint32_t total = 0;
                for (int done = 0, k = k0, rr = q0; done < tr; ++k, rr = 0) {
                    const int run = min(tr - done, inter - rr);
                    if (valid(k)) total += 2u * (uint32_t)run * (uint32_t)rga;
                    done += run;
                }
                mbar_arrive_expect_tx(full, total + xtx);
                for (int done = 0, k = k0, rr = q0; done < tr; ++k, rr = 0) {
                    const int run = min(tr - done, inter - rr);
                    if (valid(k)) {
                        const uint64_t off = (uint64_t)sids[k] * gus + (uint64_t)rr * rga;
                        const uint32_t dst = st + (uint32_t)done * (uint32_t)rga;
                        const uint32_t bytes = (uint32_t)run * (uint32_t)rga;
                        bulk_g2s(dst, pG + off, bytes, full);
                        bulk_g2s(dst + (uint32_t)aT * (uint32_t)rga, pU + off, bytes, full);
                    }
                    done += run;
                }
            } else {
                // step 3: the stage's b_T rows of every routed expert's down
                // matrix, expert k at k * b_T rows: one copy per expert
                const int64_t r0 = b_begin + (int64_t)(i - na) * bT;
                const int tr = (int)min((int64_t)bT, b_end - r0);
                const int n_seg = min(nsel, bks);
                const uint32_t bytes = (uint32_t)tr * (uint32_t)rgb;
                uint32_t total = 0;
                for (int k = 0; k < n_seg; ++k)
                    if (valid(k)) total += bytes;
                mbar_arrive_expect_tx(full, total + xtx);
                for (int k = 0; k < n_seg; ++k) {
                    if (!valid(k)) continue;
                    bulk_g2s(st + (uint32_t)(k * bT) * (uint32_t)rgb,
                             pD + (uint64_t)sids[k] * dstr + (uint64_t)r0 * rgb, bytes, full);
                }
            }
        }
        for (int j = max(0, i - S); j < i; ++j) {
            if (!mbar_wait_bounded_block(full0 + 8u * (uint32_t)(j % S), (uint32_t)((j / S) & 1))) {
                atomicOr(p.err, DEVERR_DRAIN);
                break;
            }
        }
        return;
    }

    // -------------------------------------------------------- consumers --
    const Q4kSel sel = q4k_sel(lane & 3);
    bool dead = false;
    int i = 0;
    auto wait_stage = [&](int slot, int i_) {
        if (!dead && !__all_sync(0xFFFFFFFFu, mbar_wait_bounded_block(full0 + 8u * (uint32_t)slot, (uint32_t)((i_ / S) & 1)))) {
            if (lane == 0) {
                atomicOr(p.err, DEVERR_TIMEOUT);
                *abort_flag = 1;
            }
            dead = true;
        }
    };
    {
        // ---- step 2: SwiGLU rows
        sk_stage_x<false>(xs, p.x, 1, p.hidden >> 2, 0);
        named_bar_sync(1, SK_NC * 32);
        const int nk = p.a_ksegs;
        const int ks = warp % nk, rs = warp / nk;
        const int seg_cols = min(SK_SEG, p.hidden - ks * SK_SEG);
        float2 xr[16][2];
        float xsa = 0.f, xsb = 0.f;
        rw_load_x_smem<FMT>(xs, ks, seg_cols, lane, xr, xsa, xsb);
        auto xp = [&](int gq, float2 &x02, float2 &x13) {
            x02 = xr[gq][0];
            x13 = xr[gq][1];
        };
        const bool have = 64 * (lane + 1) <= seg_cols;
        const uint32_t rb = (uint32_t)p.gu_row_bytes;
        uint32_t slice = (uint32_t)ks * (uint32_t)p.a_seg_bytes;
        slice += lane_slice_off<FMT>(lane);
        const uint32_t gst = (uint32_t)p.a_T * rb;        // the up rows follow the gate rows
        // a stage gives row slot rs rows rs*R..; a short stage (no more rows
        // than row slots: the last one of a CTA with a remainder unit) one row
        // each, so that one warp does not decode R rows while the others wait
        // at the grid barrier.  K-segment partials stay indexed by slot.
        const int nrs = p.a_T / R;                         // row slots
        constexpr int V = 2 * R;
        constexpr int SH = 5 - Log2<V>::v;
        const bool leader = (lane & ((1 << SH) - 1)) == 0;
        const int vg = (lane >> SH) / R, vk = (lane >> SH) % R;
        for (int64_t r0 = a_begin; r0 < a_end; r0 += p.a_T, ++i) {
            const int slot = i % S;
            const uint32_t st = ring + (uint32_t)slot * pitch;
            const int tr = (int)min((int64_t)p.a_T, a_end - r0);
            const bool spread = tr <= nrs;
            const int rl = spread ? rs : rs * R;
            const int ra = spread ? (rs < tr ? 1 : 0) : min(R, tr - rl);
            const bool rowok = ra > 0 && valid((int)(r0 + rl) / p.inter);
            wait_stage(slot, i);
            float acc[V];
#pragma unroll
            for (int j = 0; j < V; ++j) acc[j] = 0.f;
            QMV_SK_ROWS_PRAGMA
            for (int j = 0; j < V; ++j) {            // j = g * R + k
                const int k = j % R;
                float d = 0.f;
                if (!dead && rowok && have && k < ra) {
                    const uint32_t a = st + slice + (uint32_t)(rl + k) * rb + (uint32_t)(j / R) * gst;
                    d = lane_dot<FMT>(a, lane, sel, xp, xsa, xsb);
                }
#pragma unroll
                for (int j2 = 0; j2 < V; ++j2)
                    if (j2 == j) acc[j2] = d;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty0 + 8u * (uint32_t)slot);
            warp_transpose_reduce<V>(acc, lane);
            const int64_t row = r0 + rl + vk;
            if (nk == 1) {
                const float u = __shfl_down_sync(0xFFFFFFFFu, acc[0], R << SH);
                if (leader && vg == 0 && vk < ra) p.h[row] = rowok ? acc[0] / (1.0f + expf(-acc[0])) * u : 0.f;
            } else {
                const uint32_t pb = part0 + (uint32_t)(i & 1) * (uint32_t)(SK_PART / 2);
                if (leader) sts_f32(pb + 4u * (uint32_t)(((rs * R + vk) * 2 + vg) * nk + ks), acc[0]);
                named_bar_sync(2 + rs, 32 * nk);
                if (ks == 0 && leader && vg == 0 && vk < ra) {
                    float s0 = 0.f, s1 = 0.f;
                    const uint32_t e0 = pb + 4u * (uint32_t)((rs * R + vk) * 2 * nk);
                    for (int k2 = 0; k2 < nk; ++k2) {
                        s0 += lds_f32(e0 + 4u * (uint32_t)k2);
                        s1 += lds_f32(e0 + 4u * (uint32_t)(nk + k2));
                    }
                    p.h[row] = rowok ? s0 / (1.0f + expf(-s0)) * s1 : 0.f;
                }
            }
        }
    }
    // ---- grid barrier: every CTA's h rows are written
    named_bar_sync(1, SK_NC * 32);
    if (threadIdx.x == 0) {
        asm volatile("red.release.gpu.global.add.u32 [%0], 1;" :: "l"(p.sync) : "memory");
        const uint64_t t0 = global_timer_ns();
        for (uint32_t n = 0;; ++n) {
            unsigned v;
            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p.sync) : "memory");
            if (v >= gridDim.x) break;
            if ((n & 63u) == 63u && global_timer_ns() - t0 > 1000000000ull) {
                atomicOr(p.err, DEVERR_TIMEOUT);
                break;
            }
        }
    }
    named_bar_sync(1, SK_NC * 32);
    {
        // ---- step 3: y = sum_k g_k D_k h_k; K-segment ks is routed expert ks
        const int n_xrow = min(p.n_sel, p.b_ksegs);
        sk_stage_x<true>(xs, p.h, n_xrow, p.inter >> 2, p.inter);
        named_bar_sync(1, SK_NC * 32);
        const int nk = p.b_ksegs;
        const int ks = warp % nk, rs = warp / nk;
        const int seg_cols = ks < p.n_sel && valid(ks) ? p.inter : 0;
        float2 xr[16][2];
        float xsa = 0.f, xsb = 0.f;
        rw_load_x_smem<FMT>(xs, ks, seg_cols, lane, xr, xsa, xsb);
        auto xp = [&](int gq, float2 &x02, float2 &x13) {
            x02 = xr[gq][0];
            x13 = xr[gq][1];
        };
        const bool have = 64 * (lane + 1) <= seg_cols;
        const uint32_t rb = (uint32_t)p.d_row_bytes;
        uint32_t slice = (uint32_t)(ks * p.b_T) * rb;
        slice += lane_slice_off<FMT>(lane);
        const int nrs = p.b_T / R;
        constexpr int SH = 5 - Log2<R>::v;
        const bool leader = (lane & ((1 << SH) - 1)) == 0;
        const int vk = lane >> SH;
        for (int64_t r0 = b_begin; r0 < b_end; r0 += p.b_T, ++i) {
            const int slot = i % S;
            const uint32_t st = ring + (uint32_t)slot * pitch;
            const int tr = (int)min((int64_t)p.b_T, b_end - r0);
            const bool spread = tr <= nrs;
            const int rl = spread ? rs : rs * R;
            const int ra = spread ? (rs < tr ? 1 : 0) : min(R, tr - rl);
            wait_stage(slot, i);
            float acc[R];
#pragma unroll
            for (int k = 0; k < R; ++k) acc[k] = 0.f;
            QMV_SK_ROWS_PRAGMA
            for (int k = 0; k < R; ++k) {
                float d = 0.f;
                if (!dead && have && k < ra) {
                    const uint32_t a = st + slice + (uint32_t)(rl + k) * rb;
                    d = lane_dot<FMT>(a, lane, sel, xp, xsa, xsb);
                }
#pragma unroll
                for (int k2 = 0; k2 < R; ++k2)
                    if (k2 == k) acc[k2] = d;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty0 + 8u * (uint32_t)slot);
            warp_transpose_reduce<R>(acc, lane);
            const int64_t row = r0 + rl + vk;
            const uint32_t pb = part0 + (uint32_t)(i & 1) * (uint32_t)(SK_PART / 2);
            if (leader) sts_f32(pb + 4u * (uint32_t)((rs * R + vk) * nk + ks), acc[0]);
            named_bar_sync(2 + rs, 32 * nk);
            if (ks == 0 && leader && vk < ra) {
                float s0 = 0.f;
                for (int k2 = 0; k2 < nk; ++k2) s0 = fmaf(wseg[k2], lds_f32(pb + 4u * (uint32_t)((rs * R + vk) * nk + k2)), s0);
                p.y[row] = s0;
            }
        }
    }
    // the last CTA to leave puts the barrier words back to zero for the next launch
    named_bar_sync(1, SK_NC * 32);
    if (threadIdx.x == 0) {
        const unsigned old = atomicAdd(p.sync + 1, 1u);
        if (old == gridDim.x - 1u) {
            atomicExch(p.sync, 0u);
            atomicExch(p.sync + 1, 0u);
        }
    }
}

template <int FMT>
cudaError_t launch_skm(const SkMoeParams &p, int R, dim3 grid, size_t smem, cudaStream_t stream);

}  // namespace qmv
