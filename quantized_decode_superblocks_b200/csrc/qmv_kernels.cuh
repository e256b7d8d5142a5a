// qmv_kernels.cuh -- the sm_100a quantized matvec pipeline kernel, the MoE
// router and the dequant-only kernel.
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
//   * Each CTA owns a contiguous range of output rows.  Warp NC is the
//     producer: it streams the range's packed blocks, one tile (T rows x one
//     K-chunk, for every group) per stage, into a ring of shared-memory stages
//     with 1-D bulk async copies that complete on an mbarrier (or, when rows
//     are not 16-byte aligned, with plain 16-bit copies).
//   * Warps 0..NC-1 consume: each owns R "units" (a row of one group) per tile;
//     lane l takes the 32-weight slices l, l+32, ... of each unit, decodes them
//     in registers and accumulates f32 FMAs against x.  x comes from registers
//     (one token, rows of <= 2048 weights) or through the read-only cache.
//   * After a row's last K-chunk, one multi-row butterfly reduces the warp's
//     R x NTOK partial sums and the epilogue (plain store / weighted sum over
//     groups / SiLU-gated product) writes y.  No atomics: deterministic.
//   * Every wait is bounded (about 1 s); a timeout sets QMV_DEVERR_TIMEOUT in
//     the device error word and the warp stops instead of hanging.
#pragma once

#include <cuda_runtime.h>

#include "qmv_device.cuh"

namespace qmv {

constexpr int NC = 8;                       // consumer warps
constexpr int NTHREADS = (NC + 1) * 32;     // + one producer warp
constexpr int MAX_STAGES = 8;
constexpr int MAX_GROUPS = 8;
constexpr int SMEM_HDR = 128 + NC * 32 * 4; // barriers + per-warp result scratch

enum { MODE_SEPARATE = 0, MODE_WEIGHTED = 1, MODE_SWIGLU = 2 };
enum { DEVERR_EXPERT_ID = 1, DEVERR_TIMEOUT = 2 };

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
    // tiling
    int32_t tile_rows;       // T
    int32_t G;               // groups per job
    int32_t Gp;              // power of two >= G, <= R
    int32_t n_stage;
    int32_t stage_pitch;     // bytes per stage (multiple of 128, padded)
    int32_t row_pitch;       // bytes between consecutive units' rows in a stage
    int32_t rows_per_cta;
    int32_t mode;
    int32_t tma;             // 1: bulk async copies; 0: producer-warp copies
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

// One slice (32 weights) of one unit: dispatch to the format's decode unit.
template <int FMT, int NTOK, class XF, class XS>
__device__ __forceinline__ void slice_dot(uint32_t rowp, int s, XF &&xf, XS &&xsum, float (&a)[NTOK])
{
    if (FMT == FMT_Q8_0) {
        slice_q8_0<NTOK>(rowp + 34u * (uint32_t)s, xf, a);
    } else if (FMT == FMT_Q4_K) {
        slice_q4_k<NTOK>(rowp + 144u * (uint32_t)(s >> 3), s & 7, xf, xsum, a);
    } else {
        slice_q6_k<NTOK>(rowp + 210u * (uint32_t)(s >> 3), s & 7, xf, a);
    }
}

template <int FMT, int NTOK, int R, bool XREG>
__global__ void __launch_bounds__(NTHREADS, (NTOK <= 2 ? 2 : 1)) qmv_pipeline_kernel(const __grid_constant__ Params p)
{
    constexpr int NTP = Pow2Ceil<NTOK>::v;
    constexpr int V = R * NTP;
    static_assert(V <= 32, "R * NTOK too large");
    static_assert(!XREG || NTOK == 1, "register-resident x is for one token");
    constexpr int SPL = 2;  // slices per lane when x is register resident (cols <= 2048)

    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ const uint8_t *sW[MAX_GROUPS];
    __shared__ const float *sX[MAX_GROUPS];
    __shared__ float sWgt[MAX_GROUPS];

    const int job = blockIdx.y;
    const int64_t r_begin = (int64_t)blockIdx.x * p.rows_per_cta;
    if (r_begin >= p.rows) return;                     // uniform for the whole CTA
    const int64_t r_end = min(p.rows, r_begin + (int64_t)p.rows_per_cta);
    const int T = p.tile_rows;
    const int n_rg = (int)((r_end - r_begin + T - 1) / T);
    const int n_tiles = n_rg * p.n_chunks;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t sbase = (smem_addr(smem) + 127u) & ~127u;   // the launch adds 128 spare bytes
    const uint32_t full0 = sbase, empty0 = sbase + 64u;
    const uint32_t stage0 = sbase + (uint32_t)SMEM_HDR;

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
        for (int s = 0; s < p.n_stage; ++s) {
            mbar_init(full0 + 8u * s, 1);
            mbar_init(empty0 + 8u * s, NC);
        }
        fence_mbar_init();
    }
    __syncthreads();

    const int S = p.n_stage;

    if (warp == NC) {
        // ------------------------------------------------------ producer --
        const uint64_t pol = policy_evict_first();
        int issued = 0;
        bool ok = true;
        for (int i = 0; i < n_tiles && ok; ++i) {
            const int slot = i % S;
            if (i >= S && !mbar_wait_bounded(empty0 + 8u * slot, ((i / S) - 1) & 1)) {
                if (lane == 0) atomicOr(p.err, DEVERR_TIMEOUT);
                ok = false;
                break;
            }
            const int rg = i / p.n_chunks, kc = i % p.n_chunks;
            const int64_t r0 = r_begin + (int64_t)rg * T;
            const int tr = (int)min((int64_t)T, r_end - r0);
            const int64_t coff = (int64_t)kc * p.chunk_bytes;
            const int cbytes = (kc == p.n_chunks - 1) ? p.last_chunk_bytes : p.chunk_bytes;
            const uint32_t st = stage0 + (uint32_t)slot * (uint32_t)p.stage_pitch;
            const uint32_t full = full0 + 8u * slot;
            if (p.tma) {
                if (lane == 0) {
                    uint32_t total = 0;
                    for (int g = 0; g < p.G; ++g)
                        if (sW[g]) total += (uint32_t)tr * (uint32_t)cbytes;
                    mbar_arrive_expect_tx(full, total);
                    for (int g = 0; g < p.G; ++g) {
                        const uint8_t *W = sW[g];
                        if (!W) continue;
                        if (p.n_chunks == 1) {
                            bulk_g2s(st + (uint32_t)(g * T) * (uint32_t)p.row_pitch,
                                     W + r0 * p.row_bytes, (uint32_t)tr * (uint32_t)cbytes, full, pol);
                        } else {
                            for (int rr = 0; rr < tr; ++rr)
                                bulk_g2s(st + (uint32_t)(g * T + rr) * (uint32_t)p.row_pitch,
                                         W + (r0 + rr) * p.row_bytes + coff, (uint32_t)cbytes, full, pol);
                        }
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
                __syncwarp();
                if (lane == 0) mbar_arrive(full);
            }
            issued = i + 1;
        }
        if (!ok && p.tma && lane == 0) {
            // Do not leave the CTA while issued copies may still land in shared
            // memory: wait (bounded) for the last S issued stages.
            for (int i = max(0, issued - S); i < issued; ++i)
                (void)mbar_wait_bounded(full0 + 8u * (i % S), (i / S) & 1);
        }
        return;
    }

    // ---------------------------------------------------------- consumers --
    float4 xr[XREG ? SPL : 1][8];
    float xs[XREG ? SPL : 1][2];
    if (XREG) {
#pragma unroll
        for (int q = 0; q < SPL; ++q) {
            const int s = lane + 32 * q;
            const bool have = s * 32 < p.cols;
#pragma unroll
            for (int gq = 0; gq < 8; ++gq)
                xr[q][gq] = have ? ldg4(sX[0] + slice_group_col<FMT>(s, gq)) : make_float4(0.f, 0.f, 0.f, 0.f);
            float lo = 0.f, hi = 0.f;
#pragma unroll
            for (int gq = 0; gq < 4; ++gq) {
                lo += xr[q][gq].x + xr[q][gq].y + xr[q][gq].z + xr[q][gq].w;
                hi += xr[q][gq + 4].x + xr[q][gq + 4].y + xr[q][gq + 4].z + xr[q][gq + 4].w;
            }
            xs[q][0] = lo;
            xs[q][1] = hi;
        }
    }

    const uint32_t resw = sbase + 128u + (uint32_t)warp * 128u;   // 32 floats per warp
    float acc[V];
#pragma unroll
    for (int v = 0; v < V; ++v) acc[v] = 0.f;

    for (int i = 0; i < n_tiles; ++i) {
        const int slot = i % S;
        if (!mbar_wait_bounded(full0 + 8u * slot, (i / S) & 1)) {
            if (lane == 0) atomicOr(p.err, DEVERR_TIMEOUT);
            break;
        }
        const int rg = i / p.n_chunks, kc = i % p.n_chunks;
        const int64_t r0 = r_begin + (int64_t)rg * T;
        const int tr = (int)min((int64_t)T, r_end - r0);
        const int ccols = (kc == p.n_chunks - 1) ? p.last_chunk_cols : p.chunk_cols;
        const int n_slices = ccols >> 5;
        const int col_base = kc * p.chunk_cols;
        const uint32_t st = stage0 + (uint32_t)slot * (uint32_t)p.stage_pitch;

#pragma unroll
        for (int k = 0; k < R; ++k) {
            const int u = warp * R + k;
            const int rl = u / p.Gp, g = u % p.Gp;
            if (rl >= tr || g >= p.G || sW[g] == nullptr) continue;     // warp-uniform
            const uint32_t rowp = st + (uint32_t)(g * T + rl) * (uint32_t)p.row_pitch;
            float a[NTOK];
#pragma unroll
            for (int t = 0; t < NTOK; ++t) a[t] = 0.f;
            if (XREG) {
#pragma unroll
                for (int q = 0; q < SPL; ++q) {
                    const int s = lane + 32 * q;
                    if (s < n_slices) {
                        auto xf = [&](int, int gq) { return xr[q][gq]; };
                        auto xsum = [&](int, int hh) { return xs[q][hh]; };
                        slice_dot<FMT, NTOK>(rowp, s, xf, xsum, a);
                    }
                }
            } else {
                const float *xg = sX[g] + col_base;
                for (int s = lane; s < n_slices; s += 32) {
                    auto xf = [&](int t, int gq) {
                        return ldg4(xg + (int64_t)t * p.x_tok_stride + slice_group_col<FMT>(s, gq));
                    };
                    auto xsum = [&](int t, int hh) {
                        float r = 0.f;
#pragma unroll
                        for (int gq = 0; gq < 4; ++gq) {
                            const float4 v = xf(t, gq + 4 * hh);
                            r += (v.x + v.y) + (v.z + v.w);
                        }
                        return r;
                    };
                    slice_dot<FMT, NTOK>(rowp, s, xf, xsum, a);
                }
            }
#pragma unroll
            for (int t = 0; t < NTOK; ++t) acc[k * NTP + t] += a[t];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8u * slot);

        if (kc == p.n_chunks - 1) {
            warp_transpose_reduce<V>(acc, lane);
            constexpr int SH = 5 - Log2<V>::v;
            const int idx = lane >> SH;
            const bool leader = (lane & ((1 << SH) - 1)) == 0;
            const int k = idx / NTP, t = idx % NTP;
            if (p.mode == MODE_SEPARATE) {
                const int rl = warp * R + k;
                if (leader && t < NTOK && rl < tr)
                    p.y[(int64_t)job * p.y_job_stride + (int64_t)t * p.y_tok_stride + r0 + rl] = acc[0];
            } else {
                if (leader) sts_f32(resw + 4u * (uint32_t)(k * NTP + t), acc[0]);
                __syncwarp();
                const int rows_w = R / p.Gp;
                if (lane < rows_w * NTOK) {
                    const int rr = lane / NTOK, tt = lane % NTOK;
                    const int rl = (warp * R) / p.Gp + rr;
                    if (rl < tr) {
                        if (p.mode == MODE_WEIGHTED) {
                            float out = 0.f;
                            for (int gg = 0; gg < p.G; ++gg)
                                out = fmaf(sWgt[gg], lds_f32(resw + 4u * (uint32_t)((rr * p.Gp + gg) * NTP + tt)), out);
                            p.y[(int64_t)tt * p.y_tok_stride + r0 + rl] = out;
                        } else {
                            const float uu = lds_f32(resw + 4u * (uint32_t)((rr * 2 + 0) * NTP + tt));
                            const float vv = lds_f32(resw + 4u * (uint32_t)((rr * 2 + 1) * NTP + tt));
                            const float hval = uu / (1.0f + expf(-uu)) * vv;
                            p.y[(int64_t)job * p.y_job_stride + (int64_t)tt * p.y_tok_stride + r0 + rl] = hval;
                        }
                    }
                }
                __syncwarp();
            }
#pragma unroll
            for (int v = 0; v < V; ++v) acc[v] = 0.f;
        }
    }
}

// ------------------------------------------------------------ launchers --
struct KernelChoice {
    int ntok;
    int R;
    bool xreg;
};

// Defined per format in qmv_fmt_*.cu.
template <int FMT>
cudaError_t launch_pipeline(const Params &p, const KernelChoice &kc, dim3 grid, size_t smem,
                            cudaStream_t stream);

}  // namespace qmv
