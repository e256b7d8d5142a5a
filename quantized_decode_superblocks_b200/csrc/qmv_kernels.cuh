// qmv_kernels.cuh -- the sm_100a quantized matvec pipeline kernel.
//
// One kernel template serves every matvec form of the hot path:
//   - y = W x for a (fused) projection                    (MODE_SEPARATE, 1 job)
//   - y_k = W_{ids[k]} x_k for routed experts             (MODE_SEPARATE, n_sel jobs)
//   - y = sum_k g_k W_{ids[k]} x_k                         (MODE_WEIGHTED, n_sel groups)
//   - h_k = silu(G_{ids[k]} x) * (U_{ids[k]} x)            (MODE_SWIGLU, 2 groups per job)
// for 1..8 tokens (FlareLLM：纯Rust打造的浏览器端LLM推理引擎, §推理层面的深度优化:
// fused projections, speculative multi-token verification; BebeLM：纯Rust实现的
// 端侧大模型推理引擎, §核心算子: sigmoid-routed top-4 experts).
//
// Data path (decode is memory-bandwidth bound -- BebeLM page, §性能表现):
//   * Each CTA owns a contiguous range of output rows of one job.  Its rows
//     stream through a ring of shared-memory stages: one tile (T rows x one
//     K-chunk, for every group) per stage, moved by 1-D bulk async copies that
//     complete on the stage's mbarrier (rows that are not 16-byte aligned are
//     copied by one warp with plain 16-bit accesses instead).
//   * All 8 warps compute.  A stage is refilled by the warp that finishes it
//     last (a per-stage ticket counter), so no warp idles as a producer.
//   * Warps are split as group x K-segment x row-slot.  Each warp owns R rows
//     of one group over one K-segment; lane l takes the segment's slices l,
//     l+32, ... (32 or 64 weights each), decodes them in registers and
//     accumulates packed f32 FMAs.  With one token, x for the warp's segment
//     lives in registers for the whole kernel; with several tokens each x load
//     is reused by the warp's R rows.
//   * After a row group's last K-chunk, a multi-row warp butterfly reduces the
//     partial sums; when a row is spread over several warps (K-segments or
//     groups) the partials are combined in shared memory in a fixed order.
//     No atomics on data: results are deterministic.
//   * Every wait is bounded (about 1 s); a timeout sets QMV_DEVERR_TIMEOUT in
//     the device error word and the warp stops computing, while still taking
//     part in every barrier, so the kernel always finishes.
#pragma once

#include <cuda_runtime.h>

#include "qmv_decode45.cuh"
#include "qmv_decodemt.cuh"
#include "qmv_device.cuh"

namespace qmv {

constexpr int NW = 8;                        // warps per CTA, all compute
constexpr int NTHREADS = NW * 32;
constexpr int MAX_STAGES = 8;
constexpr int MAX_GROUPS = 8;
constexpr int SMEM_TICKET = 64;              // after MAX_STAGES full barriers
constexpr int SMEM_RES = 128;                // partial-sum exchange: 2 x 256 floats
constexpr int SMEM_HDR = 128 + 2 * 256 * 4;

enum { MODE_SEPARATE = 0, MODE_WEIGHTED = 1, MODE_SWIGLU = 2 };
enum { DEVERR_EXPERT_ID = 1, DEVERR_TIMEOUT = 2, DEVERR_DRAIN = 4 };

struct Params {
    // geometry
    int64_t rows;            // output rows per job
    int64_t row_bytes;       // packed bytes of one full row
    int32_t cols;
    int32_t chunk_cols;      // weights per K-chunk (== cols when n_chunks == 1)
    int32_t chunk_bytes;     // bytes per full K-chunk of a row
    int32_t n_chunks;
    int32_t last_chunk_cols;
    int32_t last_chunk_bytes;
    // warp roles: NW = Gp * wpr * nrs
    int32_t G;               // groups per job
    int32_t Gp;              // power of two >= G
    int32_t wpr;             // warps per row of a group (K-segments)
    int32_t nrs;             // row slots
    int32_t tile_rows;       // T = nrs * R
    // pipeline
    int32_t n_stage;
    int32_t stage_pitch;     // bytes per stage (multiple of 128, padded)
    int32_t row_pitch;       // bytes between consecutive rows in a stage
    int32_t rows_per_cta;
    int32_t mode;
    int32_t tma;             // 1: bulk async copies; 0: warp copies
    int32_t x_smem;          // x staged in shared memory after the stages: every token of one
                             // group, or (one token, x in registers) every group's x
    // weights: group matrix = base + ids[idx] * expert_stride (or base)
    const uint8_t *base0;
    const uint8_t *base1;    // MODE_SWIGLU: up matrices (group 1)
    int64_t expert_stride;
    const int32_t *ids;
    int32_t n_expert;
    // activations
    const float *x;
    int64_t x_stride;        // floats between jobs (or groups in MODE_WEIGHTED)
    int64_t x_tok_stride;    // floats between tokens
    const float *gw;         // MODE_WEIGHTED: per-group weights (device) or NULL
    // outputs
    float *y;
    int64_t y_job_stride;
    int64_t y_tok_stride;
    int *err;
};

template <int N> struct Pow2Ceil { static constexpr int v = N <= 1 ? 1 : N <= 2 ? 2 : N <= 4 ? 4 : N <= 8 ? 8 : N <= 16 ? 16 : 32; };
template <int V> struct Log2 { static constexpr int v = V >= 32 ? 5 : V >= 16 ? 4 : V >= 8 ? 3 : V >= 4 ? 2 : V >= 2 ? 1 : 0; };

__device__ __forceinline__ float4 ldg4(const float *p)
{
    return __ldg(reinterpret_cast<const float4 *>(p));
}

__device__ __forceinline__ uint32_t ldg_u16(const uint8_t *p)
{
    return __ldg(reinterpret_cast<const unsigned short *>(p));
}

__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Programmatic dependent launch: let the next kernel in the stream start its
// prologue, and wait for the previous kernel's results.  Both are no-ops when
// the launch did not opt in.
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Slices (64 weights for the K-quants, 32 for Q8_0 / Q4_0) of one K-segment: a row's
// n1 slices split over wpr warps.  For the K-quants a segment starts on a
// superblock boundary (a multiple of 4 slices), so that slice s and lane
// (s mod 32) agree on which quarter of the superblock they hold: the Q4_K
// scale selectors are built from the lane.
template <int FMT>
__device__ __forceinline__ int seg_slices(int n1, int wpr)
{
    const int P = (n1 + wpr - 1) / wpr;
    return small_block<FMT>() ? P : (P + 3) & ~3;
}

// One-token slice dot product (factored form) of one row at rowp.
template <int FMT, bool XSUM_INLINE, class XP>
__device__ __forceinline__ float dot1(uint32_t rowp, int s, const Q4kSel &sel, XP &&xp, float xsa, float xsb)
{
    if (FMT == FMT_Q8_0) {
        return q8_0_dot1(rowp + 34u * (uint32_t)s, xp);
    } else if (FMT == FMT_Q4_0) {
        return q4_0_dot1(rowp + 18u * (uint32_t)s, xp);
    } else if (FMT == FMT_Q4_K) {
        return q4_k_dot1<XSUM_INLINE>(rowp + 144u * (uint32_t)(s >> 2), s & 3, sel, xp, xsa, xsb);
    } else if (FMT == FMT_Q5_K) {
        return q5_k_dot1<XSUM_INLINE>(rowp + 176u * (uint32_t)(s >> 2), s & 3, sel, xp, xsa, xsb);
    } else {
        return q6_k_dot1(rowp + 210u * (uint32_t)(s >> 2), (s >> 1) & 1, 16 * (s & 1), xp);
    }
}

// Fill stage `slot` with the tile of rows [r0, min(r0 + T, r_end)) and K-chunk
// kc.  TMA mode: called by one thread.  Copy mode: called by a whole warp.
__device__ __forceinline__ void fill_stage(const Params &p, const uint8_t *const *sW, int64_t r0, int kc,
                                           int slot, int64_t r_end, uint32_t stage0, uint32_t full0, int lane)
{
    const int T = p.tile_rows;
    const int tr = (int)min((int64_t)T, r_end - r0);
    const int cbytes = (kc == p.n_chunks - 1) ? p.last_chunk_bytes : p.chunk_bytes;
    const int64_t coff = (int64_t)kc * p.chunk_bytes;
    const uint32_t st = stage0 + (uint32_t)slot * (uint32_t)p.stage_pitch;
    const uint32_t full = full0 + 8u * (uint32_t)slot;
    if (p.tma) {
        uint32_t total = 0;
        for (int g = 0; g < p.G; ++g)
            if (sW[g]) total += (uint32_t)tr * (uint32_t)cbytes;
        mbar_arrive_expect_tx(full, total);
        for (int g = 0; g < p.G; ++g) {
            const uint8_t *W = sW[g];
            if (!W) continue;
            if (p.n_chunks == 1) {
                bulk_g2s(st + (uint32_t)(g * T) * (uint32_t)p.row_pitch, W + r0 * p.row_bytes,
                         (uint32_t)tr * (uint32_t)cbytes, full);
            } else {
                for (int rr = 0; rr < tr; ++rr)
                    bulk_g2s(st + (uint32_t)(g * T + rr) * (uint32_t)p.row_pitch,
                             W + (r0 + rr) * p.row_bytes + coff, (uint32_t)cbytes, full);
            }
        }
    } else {
        for (int g = 0; g < p.G; ++g) {
            const uint8_t *W = sW[g];
            if (!W) continue;
            for (int rr = 0; rr < tr; ++rr) {
                const uint8_t *src = W + (r0 + rr) * p.row_bytes + coff;
                const uint32_t dst = st + (uint32_t)(g * T + rr) * (uint32_t)p.row_pitch;
#pragma unroll 4
                for (int o = 2 * lane; o < cbytes; o += 64) sts_u16(dst + o, ldg_u16(src + o));
            }
        }
        __threadfence_block();
        __syncwarp();
        if (lane == 0) mbar_arrive(full);
    }
}

// The whole pipeline for CTA `cta` of job `job` of one matvec launch.
template <int FMT, int NTOK, int R, bool XREG>
__device__ __forceinline__ void qmv_pipeline_body(const Params &p, const int cta, const int job)
{
    constexpr int NTP = Pow2Ceil<NTOK>::v;
    constexpr int V = R * NTP;
    static_assert(V <= 32, "R * NTOK too large");
    static_assert(!XREG || NTOK == 1, "register-resident x is for one token");
    constexpr int SPL1 = small_block<FMT>() ? 2 : 1;           // register-resident slices per lane
    constexpr int NG1 = Slice1<FMT>::G;

    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ const uint8_t *sW[MAX_GROUPS];
    __shared__ const float *sX[MAX_GROUPS];
    __shared__ float sWgt[MAX_GROUPS];

    const int64_t r_begin = (int64_t)cta * p.rows_per_cta;
    if (r_begin >= p.rows) return;                     // uniform for the whole CTA
    const int64_t r_end = min(p.rows, r_begin + (int64_t)p.rows_per_cta);
    const int T = p.tile_rows;
    const int n_rg = (int)((r_end - r_begin + T - 1) / T);
    const int n_tiles = n_rg * p.n_chunks;
    const int S = p.n_stage;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t sraw = smem_addr(smem);
    const uint32_t sbase = (sraw + 127u) & ~127u;      // the launch adds 128 spare bytes
    const uint32_t full0 = sbase;
    uint32_t *const ticket = reinterpret_cast<uint32_t *>(smem + (sbase - sraw) + SMEM_TICKET);
    const uint32_t res0 = sbase + SMEM_RES;
    const uint32_t stage0 = sbase + (uint32_t)SMEM_HDR;

    if (p.ids != nullptr || p.gw != nullptr) pdl_wait();   // ids / weights may come from the previous kernel
    if (tid < p.G) {
        const int g = tid;
        const int idx = (p.mode == MODE_WEIGHTED) ? g : job;
        const uint8_t *b = (p.mode == MODE_SWIGLU && g == 1) ? p.base1 : p.base0;
        const uint8_t *W = b;
        if (p.ids) {
            const int e = p.ids[idx];
            if (e < 0 || e >= p.n_expert) {
                W = nullptr;
                atomicOr(p.err, DEVERR_EXPERT_ID);
            } else {
                W = b + (int64_t)e * p.expert_stride;
            }
        }
        sW[g] = W;
        sX[g] = p.x + (int64_t)idx * p.x_stride;
        sWgt[g] = (p.mode == MODE_WEIGHTED && p.gw) ? p.gw[g] : 1.0f;
    }
    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full0 + 8u * s, 1);
            ticket[s] = 0u;
        }
        fence_mbar_init();
    }
    __syncthreads();
    pdl_launch_dependents();

    // initial fill of the ring (weights only: no dependence on earlier kernels);
    // meanwhile the other warps load x
    if ((p.tma && tid == 0) || (!p.tma && warp == 0)) {
        int64_t fr0 = r_begin;
        int fkc = 0;
        for (int i = 0; i < min(S, n_tiles); ++i) {
            fill_stage(p, sW, fr0, fkc, i, r_end, stage0, full0, lane);
            if (++fkc == p.n_chunks) { fkc = 0; fr0 += T; }
        }
    }

    // warp roles
    const int g = warp % p.Gp;
    const int ks = (warp / p.Gp) % p.wpr;
    const int rs = warp / (p.Gp * p.wpr);
    const bool active = g < p.G && sW[g] != nullptr;
    const Q4kSel sel = q4k_sel(lane & 3);

    pdl_wait();                                   // x is the previous kernel's output

    // x staged once per CTA in shared memory (swizzled): every token of one
    // group, or (one token) every group's x -- one L2 read per CTA instead of
    // one per warp, which queues behind the weight copies in flight
    const uint32_t xsm = stage0 + (uint32_t)S * (uint32_t)p.stage_pitch;
    const int nf = p.cols >> 2;                   // float4 groups per row of x
    if (p.x_smem) {
        const int nrow = NTOK > 1 ? NTOK : p.G;
        for (int idx = tid; idx < nrow * nf; idx += NTHREADS) {
            const int t = idx / nf, f = idx - t * nf;
            const float *src = NTOK > 1 ? sX[0] + (int64_t)t * p.x_tok_stride : sX[t];
            sts_f4(xsm + 16u * (uint32_t)(t * nf + (int)xs_swizzle((uint32_t)f)), ldg4(src + 4 * f));
        }
        __syncthreads();
    }

    // one token: this warp's x slices in registers for the whole kernel
    float2 xr[XREG ? SPL1 : 1][XREG ? NG1 : 1][2];
    float xsa[XREG ? SPL1 : 1], xsb[XREG ? SPL1 : 1];
    if (XREG) {
        const int n1 = p.cols / Slice1<FMT>::W;
        const int P = seg_slices<FMT>(n1, p.wpr);
#pragma unroll
        for (int q = 0; q < SPL1; ++q) {
            const int j = lane + 32 * q;
            const int s = ks * P + j;
            const bool have = active && j < P && s < n1;
            float2 sa = make_float2(0.f, 0.f), sbv = make_float2(0.f, 0.f);
#pragma unroll
            for (int gq = 0; gq < NG1; ++gq) {
                const int col = slice1_group_col<FMT>(s, gq);
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                if (have)
                    v = p.x_smem ? lds_f4(xsm + 16u * (uint32_t)(g * nf + (int)xs_swizzle((uint32_t)col >> 2)))
                                 : ldg4(sX[g] + col);
                xr[q][gq][0] = make_float2(v.x, v.z);
                xr[q][gq][1] = make_float2(v.y, v.w);
                if (gq < NG1 / 2) sa = f2add(sa, f2add(xr[q][gq][0], xr[q][gq][1]));
                else sbv = f2add(sbv, f2add(xr[q][gq][0], xr[q][gq][1]));
            }
            xsa[q] = sa.x + sa.y;
            xsb[q] = sbv.x + sbv.y;
        }
    }

    float acc[V];
#pragma unroll
    for (int v = 0; v < V; ++v) acc[v] = 0.f;
    float2 accmt[NTOK > 1 ? R : 1][NTOK > 1 ? NTOK : 1];
#pragma unroll
    for (int k = 0; k < (NTOK > 1 ? R : 1); ++k)
#pragma unroll
        for (int t = 0; t < (NTOK > 1 ? NTOK : 1); ++t) accmt[k][t] = make_float2(0.f, 0.f);

    // slice geometry of a full and of the last K-chunk
    const int n1_full = p.chunk_cols / Slice1<FMT>::W;
    const int n1_last = p.last_chunk_cols / Slice1<FMT>::W;
    const int P_full = seg_slices<FMT>(n1_full, p.wpr);
    const int P_last = seg_slices<FMT>(n1_last, p.wpr);

    // tile i: stage slot, ring round, K-chunk, first row, row-group parity --
    // advanced incrementally (no divisions in the loop); f_*: the tile i + S
    // that refills the slot once every warp has released it
    bool dead = false;
    int slot = 0, round = 0, kc = 0, rgp = 0;
    int64_t r0 = r_begin;
    int f_kc = S % p.n_chunks;
    int64_t f_r0 = r_begin + (int64_t)(S / p.n_chunks) * T;
    for (int i = 0; i < n_tiles; ++i) {
        if (!dead && !mbar_wait_bounded(full0 + 8u * (uint32_t)slot, (uint32_t)(round & 1))) {
            if (lane == 0) atomicOr(p.err, DEVERR_TIMEOUT);
            dead = true;
        }
        const bool lastc = kc == p.n_chunks - 1;
        const int tr = (int)min((int64_t)T, r_end - r0);
        const int n1 = lastc ? n1_last : n1_full;          // slices of this chunk
        const int P = lastc ? P_last : P_full;             // slices of one K-segment
        const int col_base = kc * p.chunk_cols;
        const uint32_t st = stage0 + (uint32_t)slot * (uint32_t)p.stage_pitch;
        const int s_end = min(n1, (ks + 1) * P);

        if (active && !dead) {
            if constexpr (NTOK == 1) {
#pragma unroll
                for (int k = 0; k < R; ++k) {
                    const int rl = rs * R + k;
                    if (rl >= tr) continue;                     // warp-uniform
                    const uint32_t rowp = st + (uint32_t)(g * T + rl) * (uint32_t)p.row_pitch;
                    float a = 0.f;
                    if (XREG) {
#pragma unroll
                        for (int q = 0; q < SPL1; ++q) {
                            const int s = ks * P + lane + 32 * q;
                            if (lane + 32 * q < P && s < n1) {
                                auto xp = [&](int gq, float2 &x02, float2 &x13) {
                                    x02 = xr[q][gq][0];
                                    x13 = xr[q][gq][1];
                                };
                                a += dot1<FMT, false>(rowp, s, sel, xp, xsa[q], xsb[q]);
                            }
                        }
                    } else {
                        const float *xg = sX[g] + col_base;
                        for (int s = ks * P + lane; s < s_end; s += 32) {
                            auto xp = [&](int gq, float2 &x02, float2 &x13) {
                                const float4 v = ldg4(xg + slice1_group_col<FMT>(s, gq));
                                x02 = make_float2(v.x, v.z);
                                x13 = make_float2(v.y, v.w);
                            };
                            a += dot1<FMT, true>(rowp, s, sel, xp, 0.f, 0.f);
                        }
                    }
                    acc[k] += a;
                }
            } else {
                uint32_t rowp[R];
#pragma unroll
                for (int k = 0; k < R; ++k) {
                    const int rl = rs * R + k;
                    // rows past the tile are recomputed from row 0 and never stored
                    rowp[k] = st + (uint32_t)(g * T + (rl < tr ? rl : 0)) * (uint32_t)p.row_pitch;
                }
                const float *xg = sX[g] + col_base;
                auto xl_g = [&](int t, int col) { return ldg4(xg + (int64_t)t * p.x_tok_stride + col); };
                auto xl_s = [&](int t, int col) {
                    return lds_f4(xsm + 16u * (uint32_t)(t * nf + (int)xs_swizzle((uint32_t)col >> 2)));
                };
                auto slices = [&](auto &&xl) {
                    for (int s = ks * P + lane; s < s_end; s += 32) {
                        uint32_t bp[R];
                        if (FMT == FMT_Q8_0) {
#pragma unroll
                            for (int k = 0; k < R; ++k) bp[k] = rowp[k] + 34u * (uint32_t)s;
                            q8_0_slice_mt<NTOK, R>(bp, 32 * s, xl, accmt);
                        } else if (FMT == FMT_Q4_0) {
#pragma unroll
                            for (int k = 0; k < R; ++k) bp[k] = rowp[k] + 18u * (uint32_t)s;
                            q4_0_slice_mt<NTOK, R>(bp, 32 * s, xl, accmt);
                        } else if (FMT == FMT_Q4_K) {
#pragma unroll
                            for (int k = 0; k < R; ++k) bp[k] = rowp[k] + 144u * (uint32_t)(s >> 2);
                            q4_k_slice_mt<NTOK, R>(bp, s & 3, sel, 256 * (s >> 2) + 64 * (s & 3), xl, accmt);
                        } else if (FMT == FMT_Q5_K) {
#pragma unroll
                            for (int k = 0; k < R; ++k) bp[k] = rowp[k] + 176u * (uint32_t)(s >> 2);
                            q5_k_slice_mt<NTOK, R>(bp, s & 3, sel, 256 * (s >> 2) + 64 * (s & 3), xl, accmt);
                        } else {
#pragma unroll
                            for (int k = 0; k < R; ++k) bp[k] = rowp[k] + 210u * (uint32_t)(s >> 2);
                            const int h = (s >> 1) & 1, l0 = 16 * (s & 1);
                            q6_k_slice_mt<NTOK, R>(bp, h, l0, 256 * (s >> 2) + 128 * h + l0, xl, accmt);
                        }
                    }
                };
                if (p.x_smem) slices(xl_s);
                else slices(xl_g);
            }
        }

        // release the stage; the last warp to do so refills it with tile i + S
        __syncwarp();
        uint32_t tk = 0;
        if (lane == 0) {
            __threadfence_block();
            tk = atomicAdd(&ticket[slot], 1u);
        }
        tk = __shfl_sync(0xFFFFFFFFu, tk, 0);
        if (tk == (uint32_t)(NW * (round + 1) - 1) && i + S < n_tiles) {
            __threadfence_block();
            if (p.tma) {
                if (lane == 0) {
                    fence_proxy_async_smem();
                    fill_stage(p, sW, f_r0, f_kc, slot, r_end, stage0, full0, 0);
                }
            } else {
                fill_stage(p, sW, f_r0, f_kc, slot, r_end, stage0, full0, lane);
            }
        }

        if (lastc) {
            if constexpr (NTOK > 1) {
#pragma unroll
                for (int k = 0; k < R; ++k)
#pragma unroll
                    for (int t = 0; t < NTOK; ++t) {
                        acc[k * NTP + t] = accmt[k][t].x + accmt[k][t].y;
                        accmt[k][t] = make_float2(0.f, 0.f);
                    }
            }
            warp_transpose_reduce<V>(acc, lane);
            constexpr int SH = 5 - Log2<V>::v;
            const int idx = lane >> SH;
            const bool leader = (lane & ((1 << SH) - 1)) == 0;
            const int k = idx / NTP, t = idx % NTP;
            if (p.Gp * p.wpr == 1) {
                const int rl = rs * R + k;
                if (leader && t < NTOK && rl < tr)   // one warp per row: MODE_SEPARATE or one weighted group
                    p.y[(int64_t)job * p.y_job_stride + (int64_t)t * p.y_tok_stride + r0 + rl] =
                        p.mode == MODE_WEIGHTED ? sWgt[0] * acc[0] : acc[0];
            } else {
                // partials of (warp, k, t) -> shared memory; one thread per (row, token) combines
                const uint32_t buf = res0 + (uint32_t)rgp * 1024u;
                if (leader) sts_f32(buf + 4u * (uint32_t)((warp * R + k) * NTP + t), acc[0]);
                __syncthreads();
                if (tid < T * NTOK) {
                    const int rl = tid / NTOK, tt = tid % NTOK;
                    const int rsl = rl / R, kl = rl % R;
                    if (rl < tr) {
                        float sg[MAX_GROUPS];
#pragma unroll
                        for (int gg = 0; gg < MAX_GROUPS; ++gg) {
                            float v = 0.f;
                            if (gg < p.G) {
                                for (int kk = 0; kk < p.wpr; ++kk) {
                                    const int w = gg + p.Gp * (kk + p.wpr * rsl);
                                    v += lds_f32(buf + 4u * (uint32_t)((w * R + kl) * NTP + tt));
                                }
                            }
                            sg[gg] = v;
                        }
                        float out;
                        if (p.mode == MODE_WEIGHTED) {
                            out = 0.f;
#pragma unroll
                            for (int gg = 0; gg < MAX_GROUPS; ++gg)
                                if (gg < p.G) out = fmaf(sWgt[gg], sg[gg], out);
                        } else if (p.mode == MODE_SWIGLU) {
                            out = sg[0] / (1.0f + expf(-sg[0])) * sg[1];
                        } else {
                            out = sg[0];
                        }
                        p.y[(int64_t)job * p.y_job_stride + (int64_t)tt * p.y_tok_stride + r0 + rl] = out;
                    }
                }
            }
#pragma unroll
            for (int v = 0; v < V; ++v) acc[v] = 0.f;
        }

        if (++slot == S) { slot = 0; ++round; }
        if (++kc == p.n_chunks) { kc = 0; r0 += T; rgp ^= 1; }
        if (++f_kc == p.n_chunks) { f_kc = 0; f_r0 += T; }
    }
}

template <int FMT, int NTOK, int R, bool XREG>
__global__ void __launch_bounds__(NTHREADS, (NTOK <= 2 ? 2 : 1)) qmv_pipeline_kernel(const __grid_constant__ Params p)
{
    qmv_pipeline_body<FMT, NTOK, R, XREG>(p, (int)blockIdx.x, (int)blockIdx.y);
}

// Several independent matvecs in one launch: task t owns CTAs
// [cta_begin[t], cta_begin[t+1]).
constexpr int MAX_MULTI = 64;
struct MultiParams {
    int32_t n;
    int32_t cta_begin[MAX_MULTI + 1];
    Params p[MAX_MULTI];
};

template <int FMT, int NTOK, int R, bool XREG>
__global__ void __launch_bounds__(NTHREADS, (NTOK <= 2 ? 2 : 1)) qmv_multi_kernel(const __grid_constant__ MultiParams mp)
{
    const int b = (int)blockIdx.x;
    int t = 0;
    while (t + 1 < mp.n && b >= mp.cta_begin[t + 1]) ++t;
    qmv_pipeline_body<FMT, NTOK, R, XREG>(mp.p[t], b - mp.cta_begin[t], 0);
}

// ------------------------------------------------------------ launchers --
struct KernelChoice {
    int ntok;
    int R;
    bool xreg;
    bool pdl;     // launch with programmatic stream serialization
};

// Defined per format in qmv_fmt_*.cu.
template <int FMT>
cudaError_t launch_pipeline(const Params &p, const KernelChoice &kc, dim3 grid, size_t smem,
                            cudaStream_t stream);
template <int FMT>
cudaError_t launch_multi(const MultiParams &mp, const KernelChoice &kc, int grid, size_t smem,
                         cudaStream_t stream);

}  // namespace qmv
