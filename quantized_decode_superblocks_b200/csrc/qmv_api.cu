// qmv_api.cu -- the C ABI of libqmv.so (declared in include/qmv.h): host-side
// argument validation, launch planning and the launches themselves.  Nothing
// here allocates device memory; every buffer is the caller's.
#include <algorithm>
#include <climits>
#include <atomic>
#include <mutex>
#include <type_traits>
#include <vector>

#include "../../include/qmv.h"
#include "qmv_misc.cuh"
#include "qmv_rw.cuh"
#include "qmv_sk.cuh"
#include "qmv_skt.cuh"
#include "qmv_tc.cuh"

namespace {

using namespace qmv;

// Sticky device error word (QMV_DEVERR_* bits), read and cleared by qmv_check.
__device__ int g_dev_err;

// Greedy argmax workspace of qmv_argmax (the layout of qmv_argmax_ws's): one
// 64-bit key per token, then one arrival counter per token; back to zero at
// the end of every call; qmv_check clears it after a device error.
__device__ unsigned long long g_amax_ws[QMV_ARGMAX_WS_BYTES / 8];

// Scratch of moe_ffn_static: the SwiGLU activations h[n_sel][inter].  Every
// device that loads the library holds one copy until the process exits.
static __device__ __align__(256) float g_static_h[QMV_STATIC_H_FLOATS];

constexpr int STAGE_MAX = 36 * 1024;       // bytes of one pipeline stage
constexpr int STAGES_BUDGET2 = 105 * 1024; // all stages of one CTA, two CTAs per SM (1-2 tokens)
constexpr int STAGES_BUDGET1 = 192 * 1024; // one CTA per SM (3-8 tokens: more registers per thread)
constexpr int64_t X_SMEM_MAX = 64 * 1024;       // several tokens: largest x staged in shared memory
constexpr int64_t X1_SMEM_MAX = 32 * 1024;      // one token: largest x (all groups) staged in shared memory
constexpr int MULTI_WAVES = 4;                   // grouped launch: CTA waves over the GPU
constexpr int64_t MULTI_MIN_CTA_BYTES = 128 * 1024;
#ifndef QMV_SMALL_CTA_BYTES
#define QMV_SMALL_CTA_BYTES (96 * 1024)
#endif
constexpr int64_t SMALL_CTA_BYTES = QMV_SMALL_CTA_BYTES;

struct DevInfo {
    int sm_count = 0;
    int smem_optin = 0;
    int *err = nullptr;
    unsigned long long *amax_key = nullptr;   // device address of g_amax_ws
    float *static_h = nullptr;   // device address of g_static_h, set up by moe_ffn_static
    bool ok = false;
};

std::mutex g_mu;
DevInfo g_dev[64];
std::atomic<int> g_fail_launches{0};
std::atomic<int> g_pdl{0};
std::atomic<unsigned> g_debug_extra_tx{0};
thread_local cudaError_t t_last_cuda = cudaSuccess;
// The kernel that served this host thread's most recent matvec call
// (QMV_KERNEL_*; test hook qmv_debug_last_kernel).
thread_local int t_last_kernel = QMV_KERNEL_NONE;

int cuda_fail(cudaError_t e)
{
    t_last_cuda = e;
    (void)cudaGetLastError();
    return QMV_ERR_CUDA;
}

int block_weights(int fmt)
{
    return (fmt == QMV_Q8_0 || fmt == QMV_Q4_0) ? 32 : (fmt == QMV_Q4_K || fmt == QMV_Q5_K || fmt == QMV_Q6_K) ? 256 : 0;
}
int block_bytes(int fmt)
{
    switch (fmt) {
    case QMV_Q8_0: return 34;
    case QMV_Q4_0: return 18;
    case QMV_Q4_K: return 144;
    case QMV_Q5_K: return 176;
    case QMV_Q6_K: return 210;
    default: return 0;
    }
}
bool fmt_ok(int fmt) { return block_bytes(fmt) != 0; }
// 32-weight blocks: a one-token lane slice of 64 columns is a block pair
bool small_blk(int fmt) { return fmt == QMV_Q8_0 || fmt == QMV_Q4_0; }
// the formats the warp-ring and tensor-core kernels are built for
bool rw_tc_fmt(int fmt) { return fmt == QMV_Q8_0 || fmt == QMV_Q4_K || fmt == QMV_Q6_K; }

// Calls f(std::integral_constant<int, FMT>) for block format fmt (validated:
// the QMV_* ids equal the kernels' FMT_* ids).
template <class F>
auto by_fmt(int fmt, F &&f)
{
    switch (fmt) {
    case QMV_Q8_0: return f(std::integral_constant<int, FMT_Q8_0>{});
    case QMV_Q4_0: return f(std::integral_constant<int, FMT_Q4_0>{});
    case QMV_Q4_K: return f(std::integral_constant<int, FMT_Q4_K>{});
    case QMV_Q5_K: return f(std::integral_constant<int, FMT_Q5_K>{});
    default: return f(std::integral_constant<int, FMT_Q6_K>{});
    }
}
bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
int pow2ceil(int v) { int p = 1; while (p < v) p <<= 1; return p; }

bool injected_failure()
{
    int n = g_fail_launches.load();
    while (n > 0) {
        if (g_fail_launches.compare_exchange_weak(n, n - 1)) return true;
    }
    return false;
}

int get_dev(DevInfo &out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        (void)cudaGetLastError();
        return QMV_ERR_DEVICE;
    }
    std::lock_guard<std::mutex> lk(g_mu);
    DevInfo &d = g_dev[dev];
    if (!d.ok) {
        int major = 0;
        if (cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaGetSymbolAddress(reinterpret_cast<void **>(&d.err), g_dev_err) != cudaSuccess ||
            cudaGetSymbolAddress(reinterpret_cast<void **>(&d.amax_key), g_amax_ws) != cudaSuccess) {
            (void)cudaGetLastError();
            return QMV_ERR_DEVICE;
        }
        if (major < 10) return QMV_ERR_DEVICE;   // built for sm_100a only
        d.ok = true;
    }
    out = d;
    return QMV_OK;
}

// Launch shape of one pipeline launch: how many rows a warp and a tile take,
// whether rows are split into K-chunks, the stage ring, and the grid.
struct Plan {
    KernelChoice kc;
    Params p;
    dim3 grid;
    size_t smem;
};

int make_plan(int fmt, int64_t rows, int64_t cols, int n_tok, int G, int n_jobs, bool /*shared_x*/,
              const DevInfo &di, Plan &pl, int64_t rows_per_cta_override = 0)
{
    const int bw = block_weights(fmt), bb = block_bytes(fmt);
    const int64_t rb = cols / bw * bb;
    const int ntp = pow2ceil(n_tok);
    const int gp = pow2ceil(G);
    const int sw = small_blk(fmt) ? 32 : 64;           // weights per lane slice
    const int64_t xcap = small_blk(fmt) ? 64 : 32;     // register-resident slices per lane x 32
    const int64_t n1 = cols / sw;
    const bool tma = (rb % 16) == 0;
    // Two CTAs per SM hide memory latency for large matrices.  A small matrix
    // (under SMALL_CTA_BYTES of weights per CTA at two per SM) instead takes
    // one CTA per SM, leaving the second slot free: with programmatic
    // dependent launch the next kernel's CTAs then start on it and prefetch
    // their weights while this kernel finishes.
    int ctas_per_sm = n_tok <= 2 ? 2 : 1;
    if (ctas_per_sm == 2) {
        const int64_t per_cta = ceil_div((int64_t)n_jobs * rows, 2LL * di.sm_count) * rb * G;
        if (per_cta < SMALL_CTA_BYTES) ctas_per_sm = 1;
    }
    const int target_ctas = ctas_per_sm * di.sm_count;
    const int64_t budget = n_tok <= 2 ? STAGES_BUDGET2 : STAGES_BUDGET1;
    const int64_t ctas_job0 = std::max<int64_t>(1, target_ctas / n_jobs);
    const int64_t rows_cta0 = rows_per_cta_override > 0 ? std::min(rows, rows_per_cta_override)
                                                         : ceil_div(rows, ctas_job0);

    // warps per row (K-segments): one token -> the fewest that keep a warp's x
    // in registers; several tokens -> segments of at most 2048 columns
    const int maxw = NW / gp;
    int wpr = 1;
    if (n_tok == 1) {
        while (wpr < maxw && ceil_div(n1, wpr) > xcap) wpr *= 2;
    } else {
        while (wpr < maxw && cols / wpr > 2048) wpr *= 2;
    }
    const int nrs = NW / (gp * wpr);

    const int rmax = n_tok == 1 ? 8 : std::min(4, 32 / ntp);
    int R = 1;
    for (int cand = rmax; cand >= 1; cand >>= 1) {
        const int64_t t = (int64_t)nrs * cand;
        if (t <= std::max<int64_t>(rows_cta0, nrs) && (int64_t)G * t * rb <= STAGE_MAX) {
            R = cand;
            break;
        }
    }
    if (R * ntp > 32) return QMV_ERR_SHAPE;
    const int T = nrs * R;

    int64_t chunk_cols = cols, chunk_bytes = rb;
    if ((int64_t)G * T * rb > STAGE_MAX) {
        const int64_t align = tma ? (fmt == QMV_Q6_K ? 2048 : 256) : (small_blk(fmt) ? 32 : 256);
        const int64_t per_row = STAGE_MAX / ((int64_t)G * T);
        const int64_t n_ch = ceil_div(rb, per_row);
        chunk_cols = ceil_div(ceil_div(cols, n_ch), align) * align;
        if (chunk_cols >= cols) chunk_cols = cols;
        chunk_bytes = chunk_cols / bw * bb;
    }
    const int64_t n_chunks = ceil_div(cols, chunk_cols);
    const int64_t last_cols = cols - (n_chunks - 1) * chunk_cols;
    const int64_t stage_bytes = (int64_t)G * T * chunk_bytes;
    const int64_t stage_pitch = ceil_div(stage_bytes + 16, 128) * 128;
    // x staged in shared memory when it fits: several tokens of one group, or
    // one token's x of every group (x then goes to registers from there)
    const bool xreg = n_tok == 1 && n_chunks == 1 && ceil_div(n1, wpr) <= xcap;
    const int64_t x_bytes = (int64_t)(n_tok > 1 ? n_tok : G) * cols * 4;
    const bool x_smem = n_chunks == 1 && x_bytes <= (n_tok > 1 ? X_SMEM_MAX : X1_SMEM_MAX) &&
                        (n_tok > 1 ? G == 1 : xreg);
    const int64_t x_area = x_smem ? ceil_div(x_bytes, 128) * 128 : 0;
    int n_stage = (int)std::min<int64_t>(MAX_STAGES, std::max<int64_t>(2, (budget - x_area) / stage_pitch));
    while (n_stage > 2 && 128 + SMEM_HDR + n_stage * stage_pitch + x_area > di.smem_optin) --n_stage;
    const int64_t smem = 128 + SMEM_HDR + n_stage * stage_pitch + x_area;   // 128: base alignment slack
    if (smem > di.smem_optin) return QMV_ERR_SHAPE;

    const int64_t rows_per_cta = std::max<int64_t>(1, rows_cta0);
    const int64_t ctas_per_job = ceil_div(rows, rows_per_cta);

    Params &p = pl.p;
    p = Params{};
    p.rows = rows;
    p.row_bytes = rb;
    p.cols = (int32_t)cols;
    p.chunk_cols = (int32_t)chunk_cols;
    p.chunk_bytes = (int32_t)chunk_bytes;
    p.n_chunks = (int32_t)n_chunks;
    p.last_chunk_cols = (int32_t)last_cols;
    p.last_chunk_bytes = (int32_t)(last_cols / bw * bb);
    p.G = G;
    p.Gp = gp;
    p.wpr = wpr;
    p.nrs = nrs;
    p.tile_rows = T;
    p.n_stage = n_stage;
    p.stage_pitch = (int32_t)stage_pitch;
    p.row_pitch = (int32_t)chunk_bytes;
    p.rows_per_cta = (int32_t)rows_per_cta;
    p.tma = tma ? 1 : 0;
    p.x_smem = x_smem ? 1 : 0;
    p.err = di.err;
    pl.kc.ntok = n_tok;
    pl.kc.R = R;
    pl.kc.xreg = xreg;
    pl.kc.pdl = g_pdl.load() != 0;
    pl.grid = dim3((unsigned)ctas_per_job, (unsigned)n_jobs);
    pl.smem = (size_t)smem;
    return QMV_OK;
}

int launch_plan(int fmt, const Plan &pl, cudaStream_t stream)
{
    t_last_kernel = QMV_KERNEL_GENERAL;
    cudaError_t e;
    e = by_fmt(fmt, [&](auto f) { return launch_pipeline<decltype(f)::value>(pl.p, pl.kc, pl.grid, pl.smem, stream); });
    if (e != cudaSuccess) return cuda_fail(e);
    return QMV_OK;
}

// ---------------------------------------------------------------------------
// Warp-private-ring kernel (one token, one matrix per task): tile = R rows x a
// K-chunk of up to 2048 columns; per warp S stages.  R and S depend only on the
// format (the bytes of a full K-chunk), so tasks of one format share them.
// Dynamic shared memory of one CTA, two per SM: (228 KB - 2 x 1 KB reserved) / 2
// = 113 KB, less the 128 bytes of alignment slack each launch adds.
constexpr int64_t RW_CTA_SMEM = 113 * 1024 - 128;
constexpr int64_t RW_CTA_SMEM_ONE = 227 * 1024 - 128;    // one CTA per SM (3-4 tokens)

struct RwGeom {
    int R = 0;
    int S = 0;
    int pitch = 0;
    size_t smem = 0;
};

// x_floats: shared-memory x (tasks longer than one K-chunk), taken from the
// stage budget.
RwGeom rw_geom(int fmt, int64_t x_floats, int n_tasks, int n_tok = 1)
{
    const int64_t cb = (RW_CK / block_weights(fmt)) * block_bytes(fmt);
    const int64_t x_area = n_tok * ceil_div(x_floats * 4, 128) * 128;
    const int64_t hdr = rw_hdr_bytes(n_tasks);
    const int64_t budget = n_tok > 2 ? RW_CTA_SMEM_ONE : RW_CTA_SMEM;   // 3+ tokens: one CTA per SM
    const int64_t per_warp = (budget - hdr - x_area) / NW;
    // the Q6_K decode and the several-token units read up to 4 bytes past a
    // slice (2-byte-aligned words): their stages carry 16 spare bytes
    const int64_t pad = (fmt == QMV_Q6_K || n_tok > 1) ? 16 : 0;
    auto pitch = [&](int R) { return ceil_div(R * cb + pad, 128) * 128; };
    auto stages = [&](int R) { return std::min<int64_t>(RW_MAX_STAGES, per_warp / pitch(R)); };
    RwGeom g;
    if (n_tok > 1) {
        // several tokens: two rows per warp share every x load; two stages
        for (int R : {2, 1}) {
            if (stages(R) >= 2 && R * pow2ceil(n_tok) <= 32) {
                g.R = R;
                g.S = (int)stages(R);
                g.pitch = (int)pitch(R);
                g.smem = (size_t)(128 + hdr + x_area + (int64_t)NW * g.S * g.pitch);
                return g;
            }
        }
        return g;
    }
    for (int want_s : {3, 2}) {
        for (int R : {4, 2, 1}) {
            if (stages(R) >= want_s) {
                g.R = R;
                g.S = (int)stages(R);
                g.pitch = (int)pitch(R);
                g.smem = (size_t)(128 + hdr + x_area + (int64_t)NW * g.S * g.pitch);
                return g;
            }
        }
    }
    return g;
}

// Whether a (rows x cols) matrix of fmt can take the warp-ring kernel: every
// bulk copy (a row, a K-chunk of a row) must be a multiple of 16 bytes, and a
// Q8_0 lane slice is a pair of blocks.
bool rw_ok(int fmt, int64_t cols)
{
    const int bw = block_weights(fmt), bb = block_bytes(fmt);
    if (!rw_tc_fmt(fmt)) return false;
    if (fmt == QMV_Q8_0 && cols % 64 != 0) return false;
    if (cols > RW_CK && cols > RW_X_SMEM_MAX) return false;     // x of a long row must fit in shared memory
    const int64_t rb = cols / bw * bb;
    const int64_t cb = (RW_CK / bw) * bb;
    const int64_t last_cols = cols - (ceil_div(cols, RW_CK) - 1) * RW_CK;
    const int64_t lb = last_cols / bw * bb;
    return rb % 16 == 0 && cb % 16 == 0 && lb % 16 == 0;
}

// Whether a single one-token matvec should take the warp-ring kernel rather
// than the general one (measured on B200).  Rows of one K-chunk: yes, except
// very tall Q4_K matrices (beyond ~32K rows the general kernel's Q4_K decode,
// with more rows in flight per warp, streams faster).  Longer rows: only for
// Q8_0 / Q6_K matrices of at most 4096 rows (taller ones run faster on the
// general kernel's register-resident K-segments).
bool rw_preferred(int fmt, int64_t rows, int64_t cols)
{
    if (!rw_ok(fmt, cols)) return false;
    if (cols <= RW_CK) return fmt != QMV_Q4_K || rows <= 32768;
    return fmt != QMV_Q4_K && rows <= 4096;
}

// Several tokens on the warp-ring kernel (measured on B200): up to four
// tokens (three and four with one CTA per SM); beyond that the general
// kernel's weight-stationary loop is faster.  Every token's x must fit in
// shared memory beside two stages per warp (n_tok x cols <= 32768 floats).
bool rw_mt_preferred(int fmt, int64_t rows, int64_t cols, int n_tok)
{
    (void)rows;
    if (n_tok > 4) return false;
    if (!rw_ok(fmt, cols) || (int64_t)n_tok * cols > 32768) return false;
    return rw_geom(fmt, cols, 1, n_tok).R > 0;
}

// Split a task's row groups over its nw warps, starting at warp rot (see
// rw_range in the kernel).
void rw_split(RwTask &t, int64_t nw, int64_t rot = 0)
{
    t.rg_q = t.n_rg / nw;
    t.rg_r = (int32_t)(t.n_rg % nw);
    t.nw = (int32_t)nw;
    t.rot = (int32_t)(rot % nw);
}

RwTask rw_task(int fmt, int R, const void *W, int64_t rows, int64_t cols, const float *x, float *y)
{
    const int bw = block_weights(fmt), bb = block_bytes(fmt);
    RwTask t{};
    t.W = static_cast<const uint8_t *>(W);
    t.x = x;
    t.y = y;
    t.rows = rows;
    t.row_bytes = cols / bw * bb;
    t.n_rg = ceil_div(rows, R);
    t.n_chunks = (int32_t)ceil_div(cols, RW_CK);
    t.chunk_bytes = (int32_t)((RW_CK / bw) * bb);
    t.last_cols = (int32_t)(cols - (int64_t)(t.n_chunks - 1) * RW_CK);
    t.last_bytes = (int32_t)(t.last_cols / bw * bb);
    if (t.n_chunks == 1) t.chunk_bytes = t.last_bytes;
    return t;
}

template <int NT>
cudaError_t rw_launch(int fmt, const RwParamsT<NT> &p, int R, dim3 grid, size_t smem, cudaStream_t st, bool pdl,
                      bool coop)
{
    switch (fmt) {
    case QMV_Q8_0: return launch_rw<FMT_Q8_0, NT>(p, R, grid, smem, st, pdl, coop);
    case QMV_Q4_K: return launch_rw<FMT_Q4_K, NT>(p, R, grid, smem, st, pdl, coop);
    case QMV_Q6_K: return launch_rw<FMT_Q6_K, NT>(p, R, grid, smem, st, pdl, coop);
    default: return cudaErrorInvalidValue;
    }
}

// One matvec on the warp-ring kernel: enough CTAs that every warp has a row
// group, at most two per SM.
int rw_single(int fmt, const void *W, int64_t rows, int64_t cols, const float *x, float *y, int n_tok,
              const DevInfo &di, cudaStream_t st)
{
    const int64_t x_floats = cols;
    const RwGeom g = rw_geom(fmt, x_floats, 1, n_tok);
    if (g.R == 0) return QMV_ERR_SHAPE;
    RwParams1 p{};
    p.n_tasks = 1;
    p.n_stage = g.S;
    p.stage_pitch = g.pitch;
    p.x_floats = (int32_t)x_floats;
    p.err = di.err;
    p.debug_extra_tx = g_debug_extra_tx.load();
    p.t[0] = rw_task(fmt, g.R, W, rows, cols, x, y);
    const int64_t per_sm = n_tok > 2 ? 1 : 2;
    const int64_t ctas = std::max<int64_t>(1, std::min<int64_t>(per_sm * di.sm_count, ceil_div(p.t[0].n_rg, NW)));
    p.cta_begin[0] = 0;
    p.cta_begin[1] = (int)ctas;
    rw_split(p.t[0], ctas * NW);
    const bool pdl = g_pdl.load() != 0;
    t_last_kernel = QMV_KERNEL_WARP_RING;
    cudaError_t e;
    if (n_tok == 1) {
        e = rw_launch(fmt, p, g.R, dim3((unsigned)ctas), g.smem, st, pdl, false);
    } else {
        switch (fmt) {
        case QMV_Q8_0: e = launch_rw_mt<FMT_Q8_0>(p, n_tok, g.R, dim3((unsigned)ctas), g.smem, st, pdl); break;
        case QMV_Q4_K: e = launch_rw_mt<FMT_Q4_K>(p, n_tok, g.R, dim3((unsigned)ctas), g.smem, st, pdl); break;
        case QMV_Q6_K: e = launch_rw_mt<FMT_Q6_K>(p, n_tok, g.R, dim3((unsigned)ctas), g.smem, st, pdl); break;
        default: e = cudaErrorInvalidValue; break;
        }
    }
    return e == cudaSuccess ? QMV_OK : cuda_fail(e);
}

// ---------------------------------------------------------------------------
// One-token streaming kernel (qmv_sk.cuh): one CTA of 12 consumer warps and a
// producer warp per SM, stages of T whole rows in up to ~226 KB of shared
// memory.
constexpr int64_t SK_CTA_SMEM = 226 * 1024;       // + the 128-byte alignment pad <= the 227 KB opt-in

struct SkGeom {
    bool ok = false;
    int R = 0, T = 0, S = 0, ksegs = 1, x_in_ring = 0;
    int64_t pitch = 0, x_off = 0;
    size_t smem = 0;
};

// K-segments per row: the smallest divisor of the consumer warps (twelve)
// that covers nseg segments (0 if none does).
int sk_ksegs(int64_t nseg)
{
    if (nseg < 1) return 0;
    for (int d = 1; d <= SK_NC; ++d)
        if (SK_NC % d == 0 && d >= nseg) return d;
    return 0;
}

// Geometry of a streaming-kernel launch.  mode SK_PLAIN: rows x cols (n_tok
// tokens: every token's x stays in shared memory after the ring); SK_SWIGLU:
// n_sel experts of inter rows x cols (gate and up); SK_GATHER: rows of n_sel
// expert segments of cols columns each.
SkGeom sk_geom(int fmt, int mode, int64_t rows, int64_t cols, int n_sel = 1, int64_t inter = 0, int n_tok = 1,
               int sms = 0)
{
    SkGeom g;
    const int bw = block_weights(fmt), bb = block_bytes(fmt);
    if (small_blk(fmt) && cols % 64 != 0) return g;      // a Q8_0 / Q4_0 lane slice is a 4-byte-aligned block pair
    const int64_t rb = cols / bw * bb;
    // GATHER: one K-segment per routed expert, each expert row at most one segment long
    const int64_t nseg = mode == SK_GATHER ? (cols <= SK_SEG ? n_sel : 0) : ceil_div(cols, SK_SEG);
    g.ksegs = sk_ksegs(nseg);
    if (g.ksegs == 0 || (mode == SK_GATHER && g.ksegs < n_sel)) return g;
    if (mode != SK_SWIGLU && (rows * rb) % 16 != 0) return g;   // the last copy ends on a 16-byte boundary
    // x staged in shared memory (GATHER: one 2048-column row per expert)
    const int64_t x_bytes = mode == SK_GATHER ? (int64_t)g.ksegs * SK_SEG * 4 : n_tok * ceil_div(cols * 4, 128) * 128;
    if (x_bytes > SK_X_MAX_BYTES || (n_tok > 1 && mode != SK_PLAIN)) return g;
    const int64_t budget = SK_CTA_SMEM - SK_HDR - SK_PART;
    // plain: four rows per warp for one token (Q8_0 2048x8192 6.9 -> 6.0 us,
    // Q6_K 128000x2048 53.3 -> 50.4 us against two) and for two tokens of a
    // K-quant, whose decode the four rows' shared x loads pay for (Q6_K
    // 128000x2048 92.3 -> 77.3 us; Q8_0 gate/up 13.0 -> 13.8 us, so not Q8_0);
    // fewer for small matrices
    const int r_max = mode == SK_PLAIN && (n_tok == 1 || (n_tok == 2 && !small_blk(fmt))) ? 4 : 2;
    int r_pref = r_max;
    if (sms > 0 && mode == SK_PLAIN && n_tok <= 2) {
        // a matrix whose share per CTA fills at most half of one stage: fewer
        // rows per warp, so that every warp gets some (Q4_K 3072x2048: 21 rows
        // a CTA on 12 warps of 2 rows rather than 6 warps of 4)
        const int64_t per_cta = ceil_div(rows, (int64_t)sms);
        while (r_pref > 1 && 2 * per_cta <= (int64_t)(SK_NC / g.ksegs) * r_pref) r_pref >>= 1;
    }
    auto fits = [&](int R) {
        if ((R * rb) % 16 != 0) return false;             // every row slot's copies 16-byte aligned
        if (mode == SK_SWIGLU && inter % R != 0) return false;   // a row slot never straddles two experts
        const int nrs = SK_NC / g.ksegs;
        const int64_t rs_bytes = (mode == SK_SWIGLU ? 2 : mode == SK_GATHER ? g.ksegs : 1) * R * rb;
        const int64_t pitch = ceil_div(nrs * rs_bytes + 16, 128) * 128;
        const bool in_ring = n_tok == 1 && x_bytes <= pitch;
        const int64_t S = std::min<int64_t>(SK_MAX_STAGES, (budget - (in_ring ? 0 : x_bytes)) / pitch);
        if (S < (R == 2 ? 3 : 2)) return false;          // four-row stages (up to 104 KB) run double-buffered
        g.R = R;
        g.T = nrs * R;
        g.S = (int)S;
        g.pitch = pitch;
        g.x_in_ring = in_ring ? 1 : 0;
        g.x_off = in_ring ? 0 : S * pitch;
        g.smem = (size_t)(128 + SK_HDR + SK_PART + S * pitch + (in_ring ? 0 : x_bytes));
        g.ok = true;
        return true;
    };
    for (int R = r_pref; R >= 1; R >>= 1)
        if (fits(R)) return g;
    for (int R = 2 * r_pref; R <= r_max; R <<= 1)       // the preferred R does not fit: a larger one may
        if (fits(R)) return g;
    return g;
}

// Fills the geometry fields of p and launches; the caller set the mode's
// pointers, rows, cols and row_bytes.
int sk_launch(int fmt, int mode, SkParams &p, const SkGeom &g, const DevInfo &di, cudaStream_t st)
{
    const int bw = block_weights(fmt), bb = block_bytes(fmt);
    const int64_t units = ceil_div(p.rows, (int64_t)g.R);
    const int64_t ctas = std::max<int64_t>(1, std::min<int64_t>(di.sm_count, units));
    p.units_q = units / ctas;
    p.units_r = (int32_t)(units % ctas);
    p.gran = g.R;
    p.ksegs = g.ksegs;
    p.seg_bytes = (int32_t)(SK_SEG / bw * bb);
    p.tile_rows = g.T;
    p.n_stage = g.S;
    p.stage_pitch = (int32_t)g.pitch;
    p.x_in_ring = g.x_in_ring;
    p.x_off = (int32_t)g.x_off;
    p.err = di.err;
    p.debug_extra_tx = g_debug_extra_tx.load();
    const bool pdl = g_pdl.load() != 0;
    t_last_kernel = QMV_KERNEL_STREAM;
    cudaError_t e;
    e = by_fmt(fmt, [&](auto f) {
        return launch_sk<decltype(f)::value>(p, mode, g.R, dim3((unsigned)ctas), g.smem, st, pdl);
    });
    return e == cudaSuccess ? QMV_OK : cuda_fail(e);
}

// Several tokens (2..SKT_MAX_NTOK) of a plain matrix on the streaming kernel's
// several-token form (qmv_skt.cuh); g from sk_geom(..., n_tok).
int skt_single(int fmt, const void *W, int64_t rows, int64_t cols, const float *x, float *y, int n_tok,
               const SkGeom &g, const DevInfo &di, cudaStream_t st)
{
    const int bw = block_weights(fmt), bb = block_bytes(fmt);
    SkParams p{};
    p.W = static_cast<const uint8_t *>(W);
    p.x = x;
    p.y = y;
    p.rows = rows;
    p.cols = (int32_t)cols;
    p.row_bytes = cols / bw * bb;
    p.n_sel = 1;
    p.x_row = (int32_t)(ceil_div(cols * 4, 128) * 128);
    const int64_t units = ceil_div(p.rows, (int64_t)g.R);
    const int64_t ctas = std::max<int64_t>(1, std::min<int64_t>(di.sm_count, units));
    p.units_q = units / ctas;
    p.units_r = (int32_t)(units % ctas);
    p.gran = g.R;
    p.ksegs = g.ksegs;
    p.seg_bytes = (int32_t)(SK_SEG / bw * bb);
    p.tile_rows = g.T;
    p.n_stage = g.S;
    p.stage_pitch = (int32_t)g.pitch;
    p.x_in_ring = 0;
    p.x_off = (int32_t)g.x_off;
    p.err = di.err;
    p.debug_extra_tx = g_debug_extra_tx.load();
    const bool pdl = g_pdl.load() != 0;
    t_last_kernel = QMV_KERNEL_STREAM;
    const cudaError_t e = by_fmt(fmt, [&](auto f) {
        return launch_skt<decltype(f)::value>(p, n_tok, g.R, dim3((unsigned)ctas), g.smem, st, pdl);
    });
    return e == cudaSuccess ? QMV_OK : cuda_fail(e);
}

int sk_single(int fmt, const void *W, int64_t rows, int64_t cols, const float *x, float *y, const SkGeom &g,
              const DevInfo &di, cudaStream_t st, int32_t *amax_idx = nullptr,
              unsigned long long *amax_key = nullptr, unsigned *amax_done = nullptr,
              const void *pf = nullptr, int64_t pf_bytes = 0)
{
    SkParams p{};
    p.pf = static_cast<const uint8_t *>(pf);
    p.pf_bytes = pf_bytes;
    p.amax_idx = amax_idx;
    p.amax_key = amax_key;
    p.amax_done = amax_done;
    p.W = static_cast<const uint8_t *>(W);
    p.x = x;
    p.y = y;
    p.rows = rows;
    p.cols = (int32_t)cols;
    p.row_bytes = cols / block_weights(fmt) * block_bytes(fmt);
    p.n_sel = 1;
    return sk_launch(fmt, SK_PLAIN, p, g, di, st);
}

// Several tokens of a Q8_0 or Q4_K matrix on the tensor-core kernel: one CTA of
// TC_WARPS warps per SM, x in shared memory when it fits next to rings of at
// least two stages, else read through L2.
struct TcGeom {
    bool ok = false;
    bool x_smem = false;
    int S = 0;
    int ksplit = 1;
    size_t smem = 0;
};

// Bytes of one row's 256-column K-chunk, and of its slot in a stage (Q6_K:
// the 16-byte-aligned 224 bytes around a 210-byte superblock, in a 240-byte
// slot whose 60-word pitch keeps the rows a quad group reads in different
// banks).
int tc_chunk_bytes(int fmt) { return fmt == QMV_Q8_0 ? TC_KCOLS / 32 * 34 : fmt == QMV_Q4_K ? 144 : 210; }
int tc_slot_bytes(int fmt) { return fmt == QMV_Q6_K ? 240 : tc_chunk_bytes(fmt); }

TcGeom tc_geom(int fmt, int64_t cols, int n_tok, const DevInfo &di)
{
    TcGeom g;
    const int tile = TC_ROWS * tc_slot_bytes(fmt);
    const int64_t kc_n = cols / TC_KCOLS;
    g.ksplit = kc_n % 8 == 0 ? 8 : kc_n % 4 == 0 ? 4 : kc_n % 2 == 0 ? 2 : 1;
    const int64_t sx = fmt == QMV_Q4_K ? ((cols + 127) & ~(int64_t)127) : 0;   // sum-x table
    const int64_t budget =
        (int64_t)std::min(di.smem_optin, 227 * 1024) - 128 - TC_BAR_BYTES - tc_part_bytes(TC_WARPS) - sx;
    int64_t xb = ((int64_t)n_tok * (cols + 4) * 4 + 127) & ~(int64_t)127;
    int64_t S = (budget - xb) / ((int64_t)TC_WARPS * tile);
    g.x_smem = S >= 2;
    if (!g.x_smem) {
        xb = 0;
        S = budget / ((int64_t)TC_WARPS * tile);
    }
    S = std::min<int64_t>(S, TC_MAX_STAGES);
    if (S < 2 || (fmt == QMV_Q6_K && !g.x_smem)) return g;
    g.S = (int)S;
    g.smem = (size_t)(128 + TC_BAR_BYTES + xb + tc_part_bytes(TC_WARPS) + sx + (int64_t)TC_WARPS * S * tile);
    g.ok = true;
    return g;
}

// Q8_0 / Q4_K with 3..8 tokens whose rows are whole 256-column K-chunks;
// Q6_K when rows are whole 2048-column runs (a multiple of 16 bytes, so a
// superblock's offset in its 16-byte-aligned slot is the same in every row).
bool tc_preferred(int fmt, int64_t rows, int64_t cols, int n_tok)
{
    const bool shape = fmt == QMV_Q6_K                        ? cols % 2048 == 0
                       : (fmt == QMV_Q8_0 || fmt == QMV_Q4_K) ? cols % TC_KCOLS == 0
                                                              : false;
    return shape && n_tok >= 3 && n_tok <= 8 && cols <= (int64_t)1 << 24 && rows <= (int64_t)INT_MAX;
}

int tc_single(int fmt, const void *W, int64_t rows, int64_t cols, const float *x, float *y, int n_tok,
              const DevInfo &di, cudaStream_t st)
{
    const TcGeom g = tc_geom(fmt, cols, n_tok, di);
    if (!g.ok) return QMV_ERR_SHAPE;
    TcParams p{};
    p.W = static_cast<const uint8_t *>(W);
    p.x = x;
    p.y = y;
    p.rows = rows;
    p.row_bytes = cols / TC_KCOLS * tc_chunk_bytes(fmt);   // Q6_K: a multiple of 16 (cols % 2048 == 0)
    p.cols = (int32_t)cols;
    p.n_tok = n_tok;
    p.kc_n = (int32_t)(cols / TC_KCOLS);
    p.chunk_bytes = tc_chunk_bytes(fmt);
    p.slot_bytes = tc_slot_bytes(fmt);
    p.ksplit = g.ksplit;
    const int64_t n_rt = ceil_div(rows, (int64_t)TC_ROWS);
    p.n_rt = (int32_t)n_rt;
    const int64_t ctas = std::max<int64_t>(1, std::min<int64_t>(n_rt, di.sm_count));
    p.rt_q = (int32_t)(n_rt / ctas);
    p.rt_r = (int32_t)(n_rt % ctas);
    p.n_stage = g.S;
    p.x_pitch = (int32_t)(cols + 4);
    p.err = di.err;
    p.debug_extra_tx = g_debug_extra_tx.load();
    const bool pdl = g_pdl.load() != 0;
    t_last_kernel = QMV_KERNEL_TENSOR_CORE;
    const cudaError_t e = fmt == QMV_Q8_0   ? launch_tc<FMT_Q8_0>(p, g.x_smem, dim3((unsigned)ctas), g.smem, st, pdl)
                          : fmt == QMV_Q4_K ? launch_tc<FMT_Q4_K>(p, g.x_smem, dim3((unsigned)ctas), g.smem, st, pdl)
                                            : launch_tc<FMT_Q6_K>(p, g.x_smem, dim3((unsigned)ctas), g.smem, st, pdl);
    return e == cudaSuccess ? QMV_OK : cuda_fail(e);
}


// In-order one-token matvecs as one streaming-kernel launch each, ordered by
// programmatic dependent launch (each kernel reads its x only after the
// previous one has finished).  Each launch, once its own weight copies are
// issued, moves the next task's weights into L2: the next launch's copies then
// come from L2 while HBM already streams the one after.  Returns QMV_ERR_SHAPE
// (nothing launched) when some task does not fit the streaming kernel.
int sk_seq(int fmt, const qmv_task *tasks, int n_tasks, const DevInfo &di, cudaStream_t st)
{
    for (int t = 0; t < n_tasks; ++t)
        if (!sk_geom(fmt, SK_PLAIN, tasks[t].rows, tasks[t].cols).ok) return QMV_ERR_SHAPE;
    const int bw = block_weights(fmt), bb = block_bytes(fmt);
    for (int t = 0; t < n_tasks; ++t) {
        const qmv_task &k = tasks[t];
        const qmv_task *nx = t + 1 < n_tasks ? &tasks[t + 1] : nullptr;
        const SkGeom g = sk_geom(fmt, SK_PLAIN, k.rows, k.cols, 1, 0, 1, di.sm_count);
        const int rc = sk_single(fmt, k.W_blocks, k.rows, k.cols, k.x, k.y, g, di, st, nullptr, nullptr, nullptr,
                                 nx ? nx->W_blocks : nullptr, nx ? nx->rows * (nx->cols / bw * bb) : 0);
        if (rc) return rc;
    }
    return QMV_OK;
}


int check_matrix(int fmt, int64_t rows, int64_t cols)
{
    if (!fmt_ok(fmt)) return QMV_ERR_FMT;
    if (rows < 1 || cols < 1 || rows > QMV_MAX_ROWS || cols > QMV_MAX_COLS || cols % block_weights(fmt) != 0)
        return QMV_ERR_SHAPE;
    return QMV_OK;
}

int argmax_check(int fmt, const void *W, int64_t rows, int64_t cols, const float *x, const float *y, int n_tok,
                 const int32_t *idx_out)
{
    if (!W || !x || !y || !idx_out) return QMV_ERR_NULL;
    const int rc = check_matrix(fmt, rows, cols);
    if (rc) return rc;
    if (rows > INT32_MAX) return QMV_ERR_SHAPE;
    if (n_tok < 1 || n_tok > QMV_MAX_NTOK) return QMV_ERR_NTOK;
    if (!aligned(W, 16) || !aligned(x, 16) || !aligned(y, 4) || !aligned(idx_out, 4)) return QMV_ERR_ALIGN;
    return QMV_OK;
}

}  // namespace

extern "C" {

size_t qmv_block_bytes(int fmt) { return (size_t)block_bytes(fmt); }
int qmv_block_weights(int fmt) { return block_weights(fmt); }

void qmv_debug_fail_next_launches(int count) { g_fail_launches.store(count > 0 ? count : 0); }

void qmv_set_pdl(int enable) { g_pdl.store(enable ? 1 : 0); }

void qmv_debug_short_copies(int bytes) { g_debug_extra_tx.store(bytes > 0 ? (unsigned)bytes : 0u); }

int qmv_get_pdl(void) { return g_pdl.load(); }

int qmv_debug_last_kernel(void) { return t_last_kernel; }

const char *qmv_last_cuda_error(void)
{
    return t_last_cuda == cudaSuccess ? "no error" : cudaGetErrorString(t_last_cuda);
}

const char *qmv_strerror(int status)
{
    switch (status) {
    case QMV_OK: return "success";
    case QMV_ERR_NULL: return "a required pointer is NULL";
    case QMV_ERR_FMT: return "unknown block format";
    case QMV_ERR_SHAPE: return "bad shape (rows/cols < 1, cols not a multiple of the block size, or too large)";
    case QMV_ERR_ALIGN: return "misaligned pointer or stride (W and x need 16 bytes, y 4 bytes)";
    case QMV_ERR_NTOK: return "n_tok outside [1, 8]";
    case QMV_ERR_NSEL: return "n_sel / top_k / n_expert outside the supported range";
    case QMV_ERR_CUDA: return "a CUDA call or kernel launch failed";
    case QMV_ERR_DEVICE: return "no usable sm_100 device, or a device-side error was recorded";
    default: return "unknown status";
    }
}

int qmv_batched(int fmt, const void *W_blocks, int64_t rows, int64_t cols, const float *x, float *y,
                int n_tok, qmv_stream_t stream)
{
    if (!W_blocks || !x || !y) return QMV_ERR_NULL;
    int rc = check_matrix(fmt, rows, cols);
    if (rc) return rc;
    if (n_tok < 1 || n_tok > QMV_MAX_NTOK) return QMV_ERR_NTOK;
    if (!aligned(W_blocks, 16) || !aligned(x, 16) || !aligned(y, 4)) return QMV_ERR_ALIGN;
    if (injected_failure()) return QMV_ERR_CUDA;
    DevInfo di;
    if ((rc = get_dev(di))) return rc;
    if (tc_preferred(fmt, rows, cols, n_tok) && tc_geom(fmt, cols, n_tok, di).ok)
        return tc_single(fmt, W_blocks, rows, cols, x, y, n_tok, di, reinterpret_cast<cudaStream_t>(stream));
    if (n_tok == 1) {
        const SkGeom g = sk_geom(fmt, SK_PLAIN, rows, cols, 1, 0, 1, di.sm_count);
        if (g.ok) return sk_single(fmt, W_blocks, rows, cols, x, y, g, di, reinterpret_cast<cudaStream_t>(stream));
    } else if (n_tok <= SKT_MAX_NTOK) {
        const SkGeom g = sk_geom(fmt, SK_PLAIN, rows, cols, 1, 0, n_tok, di.sm_count);
        if (g.ok)
            return skt_single(fmt, W_blocks, rows, cols, x, y, n_tok, g, di, reinterpret_cast<cudaStream_t>(stream));
    }
    if (n_tok == 1 ? rw_preferred(fmt, rows, cols) : rw_mt_preferred(fmt, rows, cols, n_tok))
        return rw_single(fmt, W_blocks, rows, cols, x, y, n_tok, di, reinterpret_cast<cudaStream_t>(stream));
    Plan pl;
    if ((rc = make_plan(fmt, rows, cols, n_tok, 1, 1, true, di, pl))) return rc;
    pl.p.mode = MODE_SEPARATE;
    pl.p.base0 = static_cast<const uint8_t *>(W_blocks);
    pl.p.x = x;
    pl.p.x_tok_stride = cols;
    pl.p.y = y;
    pl.p.y_tok_stride = rows;
    return launch_plan(fmt, pl, reinterpret_cast<cudaStream_t>(stream));
}

int qmv_multi(int fmt, int n_tok, const qmv_task *tasks, int n_tasks, qmv_stream_t stream)
{
    if (!tasks) return QMV_ERR_NULL;
    if (!fmt_ok(fmt)) return QMV_ERR_FMT;
    if (n_tasks < 1 || n_tasks > QMV_MAX_TASKS) return QMV_ERR_SHAPE;
    if (n_tok < 1 || n_tok > QMV_MAX_NTOK) return QMV_ERR_NTOK;
    int64_t total = 0;
    for (int t = 0; t < n_tasks; ++t) {
        const qmv_task &k = tasks[t];
        if (!k.W_blocks || !k.x || !k.y) return QMV_ERR_NULL;
        const int rc = check_matrix(fmt, k.rows, k.cols);
        if (rc) return rc;
        if (!aligned(k.W_blocks, 16) || !aligned(k.x, 16) || !aligned(k.y, 4)) return QMV_ERR_ALIGN;
        total += k.rows * (k.cols / block_weights(fmt)) * block_bytes(fmt);
    }
    if (injected_failure()) return QMV_ERR_CUDA;
    DevInfo di;
    int rc = get_dev(di);
    if (rc) return rc;
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // Every CTA streams about the same number of bytes, sized so the batch
    // takes a few waves of two CTAs per SM: small tasks get few CTAs with many
    // rows each, and all tasks' CTAs share the GPU at once.
    const int64_t per_cta = std::max<int64_t>(MULTI_MIN_CTA_BYTES,
                                              ceil_div(total, (int64_t)MULTI_WAVES * 2 * di.sm_count));
    std::vector<Plan> plans((size_t)n_tasks);
    for (int t = 0; t < n_tasks; ++t) {
        const qmv_task &k = tasks[t];
        const int64_t bytes = k.rows * (k.cols / block_weights(fmt)) * block_bytes(fmt);
        const int64_t ctas = std::max<int64_t>(1, ceil_div(bytes, per_cta));
        Plan &pl = plans[(size_t)t];
        if ((rc = make_plan(fmt, k.rows, k.cols, n_tok, 1, 1, true, di, pl, ceil_div(k.rows, ctas)))) return rc;
        pl.p.mode = MODE_SEPARATE;
        pl.p.base0 = static_cast<const uint8_t *>(k.W_blocks);
        pl.p.x = k.x;
        pl.p.x_tok_stride = k.cols;
        pl.p.y = k.y;
        pl.p.y_tok_stride = k.rows;
    }
    // one launch per kernel instance (rows per warp, x in registers), at most
    // MAX_MULTI tasks each
    std::vector<char> done((size_t)n_tasks, 0);
    static thread_local MultiParams mp;
    t_last_kernel = QMV_KERNEL_GENERAL;
    for (int t0 = 0; t0 < n_tasks; ++t0) {
        if (done[(size_t)t0]) continue;
        const KernelChoice kc = plans[(size_t)t0].kc;
        mp.n = 0;
        size_t smem = 0;
        int ctas = 0;
        for (int t = t0; t < n_tasks && mp.n < MAX_MULTI; ++t) {
            const Plan &pl = plans[(size_t)t];
            if (done[(size_t)t] || pl.kc.R != kc.R || pl.kc.xreg != kc.xreg) continue;
            done[(size_t)t] = 1;
            mp.cta_begin[mp.n] = ctas;
            mp.p[mp.n] = pl.p;
            ctas += (int)pl.grid.x;
            smem = std::max(smem, pl.smem);
            ++mp.n;
        }
        mp.cta_begin[mp.n] = ctas;
        cudaError_t e;
        e = by_fmt(fmt, [&](auto f) { return launch_multi<decltype(f)::value>(mp, kc, ctas, smem, st); });
        if (e != cudaSuccess) return cuda_fail(e);
    }
    return QMV_OK;
}

int qmv_chain(int fmt, const qmv_task *tasks, int n_tasks, qmv_stream_t stream)
{
    if (!tasks) return QMV_ERR_NULL;
    if (!fmt_ok(fmt)) return QMV_ERR_FMT;
    if (n_tasks < 1 || n_tasks > QMV_MAX_TASKS) return QMV_ERR_SHAPE;
    for (int t = 0; t < n_tasks; ++t) {
        const qmv_task &k = tasks[t];
        if (!k.W_blocks || !k.x || !k.y) return QMV_ERR_NULL;
        const int rc = check_matrix(fmt, k.rows, k.cols);
        if (rc) return rc;
        if (!aligned(k.W_blocks, 16) || !aligned(k.x, 16) || !aligned(k.y, 4)) return QMV_ERR_ALIGN;
    }
    if (injected_failure()) return QMV_ERR_CUDA;
    DevInfo di;
    int rc = get_dev(di);
    if (rc) return rc;
    rc = sk_seq(fmt, tasks, n_tasks, di, reinterpret_cast<cudaStream_t>(stream));
    if (rc != QMV_ERR_SHAPE) return rc;
    // a shape the streaming kernel does not take: one call per task, in order
    for (int t = 0; t < n_tasks; ++t) {
        const qmv_task &k = tasks[t];
        if ((rc = qmv_batched(fmt, k.W_blocks, k.rows, k.cols, k.x, k.y, 1, stream))) return rc;
    }
    return QMV_OK;
}

int qmv_f32(int fmt, const void *W_blocks, int64_t rows, int64_t cols, const float *x, float *y,
            qmv_stream_t stream)
{
    return qmv_batched(fmt, W_blocks, rows, cols, x, y, 1, stream);
}

int moe_route(const float *logits, const float *bias, int n_expert, int top_k, int32_t *ids_out,
              float *g_out, qmv_stream_t stream)
{
    if (!logits || !bias || !ids_out || !g_out) return QMV_ERR_NULL;
    if (n_expert < 1 || n_expert > QMV_MAX_EXPERTS || top_k < 1 || top_k > QMV_MAX_SEL || top_k > n_expert)
        return QMV_ERR_NSEL;
    if (!aligned(logits, 4) || !aligned(bias, 4) || !aligned(ids_out, 4) || !aligned(g_out, 4))
        return QMV_ERR_ALIGN;
    if (injected_failure()) return QMV_ERR_CUDA;
    DevInfo di;
    int rc = get_dev(di);
    if (rc) return rc;
    moe_route_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(logits, bias, n_expert, top_k,
                                                                          ids_out, g_out);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e);
    return QMV_OK;
}

int moe_qmv(int fmt, const void *expert_blocks, int64_t expert_stride_bytes, int n_expert,
            const int32_t *expert_ids, int n_sel, int64_t rows, int64_t cols, const float *x,
            int64_t x_stride, const float *gate_w, float *y, qmv_stream_t stream)
{
    if (!expert_blocks || !expert_ids || !x || !y) return QMV_ERR_NULL;
    int rc = check_matrix(fmt, rows, cols);
    if (rc) return rc;
    if (n_expert < 1 || n_expert > QMV_MAX_EXPERTS || n_sel < 1 || n_sel > QMV_MAX_SEL || n_sel > n_expert)
        return QMV_ERR_NSEL;
    const int64_t mat_bytes = rows * (cols / block_weights(fmt)) * block_bytes(fmt);
    if (expert_stride_bytes < mat_bytes || x_stride < 0) return QMV_ERR_SHAPE;
    if (!aligned(expert_blocks, 16) || expert_stride_bytes % 16 != 0 || !aligned(x, 16) ||
        x_stride % 4 != 0 || !aligned(y, 4) || !aligned(expert_ids, 4) || (gate_w && !aligned(gate_w, 4)))
        return QMV_ERR_ALIGN;
    if (injected_failure()) return QMV_ERR_CUDA;
    DevInfo di;
    if ((rc = get_dev(di))) return rc;
    Plan pl;
    const bool weighted = gate_w != nullptr;
    if ((rc = make_plan(fmt, rows, cols, 1, weighted ? n_sel : 1, weighted ? 1 : n_sel,
                        weighted ? (x_stride == 0) : true, di, pl)))
        return rc;
    Params &p = pl.p;
    p.mode = weighted ? MODE_WEIGHTED : MODE_SEPARATE;
    p.base0 = static_cast<const uint8_t *>(expert_blocks);
    p.expert_stride = expert_stride_bytes;
    p.ids = expert_ids;
    p.n_expert = n_expert;
    p.x = x;
    p.x_stride = x_stride;
    p.x_tok_stride = cols;
    p.gw = gate_w;
    p.y = y;
    p.y_job_stride = rows;
    p.y_tok_stride = rows;
    return launch_plan(fmt, pl, reinterpret_cast<cudaStream_t>(stream));
}

int moe_ffn(int fmt_gu, const void *gate_blocks, const void *up_blocks, int64_t gu_stride_bytes,
            int fmt_down, const void *down_blocks, int64_t down_stride_bytes, int n_expert,
            const int32_t *expert_ids, const float *g, int n_sel, int64_t hidden, int64_t inter,
            const float *x, float *h_scratch, float *y, qmv_stream_t stream)
{
    if (!gate_blocks || !up_blocks || !down_blocks || !expert_ids || !g || !x || !h_scratch || !y)
        return QMV_ERR_NULL;
    int rc = check_matrix(fmt_gu, inter, hidden);
    if (rc) return rc;
    if ((rc = check_matrix(fmt_down, hidden, inter))) return rc;
    if (n_expert < 1 || n_expert > QMV_MAX_EXPERTS || n_sel < 1 || n_sel > QMV_MAX_SEL || n_sel > n_expert)
        return QMV_ERR_NSEL;
    const int64_t gu_bytes = inter * (hidden / block_weights(fmt_gu)) * block_bytes(fmt_gu);
    const int64_t dn_bytes = hidden * (inter / block_weights(fmt_down)) * block_bytes(fmt_down);
    if (gu_stride_bytes < gu_bytes || down_stride_bytes < dn_bytes) return QMV_ERR_SHAPE;
    if (!aligned(gate_blocks, 16) || !aligned(up_blocks, 16) || !aligned(down_blocks, 16) ||
        gu_stride_bytes % 16 != 0 || down_stride_bytes % 16 != 0 || !aligned(x, 16) ||
        !aligned(h_scratch, 16) || !aligned(y, 4) || !aligned(expert_ids, 4) || !aligned(g, 4))
        return QMV_ERR_ALIGN;
    if (injected_failure()) return QMV_ERR_CUDA;
    DevInfo di;
    if ((rc = get_dev(di))) return rc;
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

    const SkGeom ga = sk_geom(fmt_gu, SK_SWIGLU, (int64_t)n_sel * inter, hidden, n_sel, inter);
    const SkGeom gb = sk_geom(fmt_down, SK_GATHER, hidden, inter, n_sel);
    if (ga.ok && gb.ok && (int64_t)n_sel * inter <= INT32_MAX) {
        // h_k = silu(G_k x) * (U_k x), then y = sum_k g_k D_k h_k, on the streaming kernel
        SkParams a{};
        a.W = static_cast<const uint8_t *>(gate_blocks);
        a.W2 = static_cast<const uint8_t *>(up_blocks);
        a.expert_stride = gu_stride_bytes;
        a.ids = expert_ids;
        a.n_expert = n_expert;
        a.n_sel = n_sel;
        a.inter = (int32_t)inter;
        a.cols = (int32_t)hidden;
        a.x = x;
        a.y = h_scratch;
        a.rows = (int64_t)n_sel * inter;
        a.row_bytes = hidden / block_weights(fmt_gu) * block_bytes(fmt_gu);
        if ((rc = sk_launch(fmt_gu, SK_SWIGLU, a, ga, di, st))) return rc;
        SkParams b{};
        b.W = static_cast<const uint8_t *>(down_blocks);
        b.expert_stride = down_stride_bytes;
        b.ids = expert_ids;
        b.gw = g;
        b.n_expert = n_expert;
        b.n_sel = n_sel;
        b.cols = (int32_t)inter;
        b.x = h_scratch;
        b.y = y;
        b.rows = hidden;
        b.row_bytes = inter / block_weights(fmt_down) * block_bytes(fmt_down);
        return sk_launch(fmt_down, SK_GATHER, b, gb, di, st);
    }

    // h_k = silu(G_k x) * (U_k x): two groups (gate, up) per routed expert
    Plan a;
    if ((rc = make_plan(fmt_gu, inter, hidden, 1, 2, n_sel, true, di, a))) return rc;
    a.p.mode = MODE_SWIGLU;
    a.p.base0 = static_cast<const uint8_t *>(gate_blocks);
    a.p.base1 = static_cast<const uint8_t *>(up_blocks);
    a.p.expert_stride = gu_stride_bytes;
    a.p.ids = expert_ids;
    a.p.n_expert = n_expert;
    a.p.x = x;
    a.p.x_stride = 0;
    a.p.x_tok_stride = hidden;
    a.p.y = h_scratch;
    a.p.y_job_stride = inter;
    a.p.y_tok_stride = inter;
    if ((rc = launch_plan(fmt_gu, a, st))) return rc;

    // y = sum_k g_k D_k h_k: one group per routed expert, weighted in k order
    Plan b;
    if ((rc = make_plan(fmt_down, hidden, inter, 1, n_sel, 1, false, di, b))) return rc;
    b.p.mode = MODE_WEIGHTED;
    b.p.base0 = static_cast<const uint8_t *>(down_blocks);
    b.p.expert_stride = down_stride_bytes;
    b.p.ids = expert_ids;
    b.p.n_expert = n_expert;
    b.p.x = h_scratch;
    b.p.x_stride = inter;
    b.p.x_tok_stride = inter;
    b.p.gw = g;
    b.p.y = y;
    b.p.y_tok_stride = hidden;
    return launch_plan(fmt_down, b, st);
}

int moe_ffn_routed(const float *logits, const float *bias, int n_expert, int top_k, int fmt_gu,
                   const void *gate_blocks, const void *up_blocks, int64_t gu_stride_bytes, int fmt_down,
                   const void *down_blocks, int64_t down_stride_bytes, int64_t hidden, int64_t inter,
                   const float *x, int32_t *ids_out, float *g_out, float *h_scratch, float *y, void *workspace,
                   qmv_stream_t stream)
{
    if (!logits || !bias || !gate_blocks || !up_blocks || !down_blocks || !x || !ids_out || !g_out ||
        !h_scratch || !y || !workspace)
        return QMV_ERR_NULL;
    int rc = check_matrix(fmt_gu, inter, hidden);
    if (rc) return rc;
    if ((rc = check_matrix(fmt_down, hidden, inter))) return rc;
    if (n_expert < 1 || n_expert > QMV_MAX_EXPERTS || top_k < 1 || top_k > QMV_MAX_SEL || top_k > n_expert)
        return QMV_ERR_NSEL;
    const int64_t gu_bytes = inter * (hidden / block_weights(fmt_gu)) * block_bytes(fmt_gu);
    const int64_t dn_bytes = hidden * (inter / block_weights(fmt_down)) * block_bytes(fmt_down);
    if (gu_stride_bytes < gu_bytes || down_stride_bytes < dn_bytes) return QMV_ERR_SHAPE;
    if (!aligned(logits, 4) || !aligned(bias, 4) || !aligned(gate_blocks, 16) || !aligned(up_blocks, 16) ||
        !aligned(down_blocks, 16) || gu_stride_bytes % 16 != 0 || down_stride_bytes % 16 != 0 || !aligned(x, 16) ||
        !aligned(ids_out, 4) || !aligned(g_out, 4) || !aligned(h_scratch, 16) || !aligned(y, 4) ||
        !aligned(workspace, 8))
        return QMV_ERR_ALIGN;
    if (injected_failure()) return QMV_ERR_CUDA;
    DevInfo di;
    if ((rc = get_dev(di))) return rc;
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

    // the one-launch form: both matrices of one format, expert rows of at most
    // one K-segment, the router on the device in every CTA
    const int bw = block_weights(fmt_gu), bb = block_bytes(fmt_gu);
    const int R = 2;
    const int64_t rba = hidden / bw * bb, rbb = inter / bw * bb;
    const int ka = sk_ksegs(ceil_div(hidden, SK_SEG)), kb = sk_ksegs(top_k);
    bool fused = fmt_gu == fmt_down && n_expert <= SKM_MAX_EXPERTS && inter <= SK_SEG && ka > 0 && kb >= top_k &&
                 inter % R == 0 && (R * rba) % 16 == 0 && (R * rbb) % 16 == 0 &&
                 (!small_blk(fmt_gu) || (hidden % 64 == 0 && inter % 64 == 0));
    SkMoeParams p{};
    size_t smem = 0;
    if (fused) {
        const int64_t stage_a = (int64_t)(SK_NC / ka) * 2 * R * rba, stage_b = (int64_t)(SK_NC / kb) * kb * R * rbb;
        const int64_t pitch = ceil_div(std::max(stage_a, stage_b) + 16, 128) * 128;
        const int64_t x_bytes = ceil_div(std::max<int64_t>(hidden * 4, (int64_t)kb * SK_SEG * 4), 128) * 128;
        const int64_t S = std::min<int64_t>(SK_MAX_STAGES, (SK_CTA_SMEM - SK_HDR - SK_PART - x_bytes) / pitch);
        fused = S >= 2 && x_bytes <= SK_X_MAX_BYTES;
        const int64_t ctas = di.sm_count;
        const int64_t ua = ceil_div((int64_t)top_k * inter, (int64_t)R), ub = ceil_div(hidden, (int64_t)R);
        p.logits = logits;
        p.bias = bias;
        p.ids_out = ids_out;
        p.g_out = g_out;
        p.n_expert = n_expert;
        p.n_sel = top_k;
        p.G = static_cast<const uint8_t *>(gate_blocks);
        p.U = static_cast<const uint8_t *>(up_blocks);
        p.gu_stride = gu_stride_bytes;
        p.gu_row_bytes = rba;
        p.D = static_cast<const uint8_t *>(down_blocks);
        p.d_stride = down_stride_bytes;
        p.d_row_bytes = rbb;
        p.hidden = (int32_t)hidden;
        p.inter = (int32_t)inter;
        p.x = x;
        p.h = h_scratch;
        p.y = y;
        p.a_ksegs = ka;
        p.a_seg_bytes = SK_SEG / bw * bb;
        p.a_T = (SK_NC / ka) * R;
        p.a_units_q = ua / ctas;
        p.a_units_r = (int32_t)(ua % ctas);
        p.b_ksegs = kb;
        p.b_T = (SK_NC / kb) * R;
        p.b_units_q = ub / ctas;
        p.b_units_r = (int32_t)(ub % ctas);
        p.n_stage = (int32_t)S;
        p.stage_pitch = (int32_t)pitch;
        p.x_off = (int32_t)(S * pitch);
        p.sync = static_cast<unsigned *>(workspace);
        p.err = di.err;
        p.debug_extra_tx = g_debug_extra_tx.load();
        smem = (size_t)(128 + SK_HDR + SK_PART + S * pitch + x_bytes);
    }
    if (fused) {
        t_last_kernel = QMV_KERNEL_STREAM;
        cudaError_t e;
        e = by_fmt(fmt_gu, [&](auto f) {
            return launch_skm<decltype(f)::value>(p, R, dim3((unsigned)di.sm_count), smem, st);
        });
        return e == cudaSuccess ? QMV_OK : cuda_fail(e);
    }
    // other shapes: the router, then the two-launch FFN step
    if ((rc = moe_route(logits, bias, n_expert, top_k, ids_out, g_out, stream))) return rc;
    return moe_ffn(fmt_gu, gate_blocks, up_blocks, gu_stride_bytes, fmt_down, down_blocks, down_stride_bytes,
                   n_expert, ids_out, g_out, top_k, hidden, inter, x, h_scratch, y, stream);
}

int moe_ffn_static(int fmt_gu, const void *gate_blocks, const void *up_blocks, int64_t gu_stride_bytes,
                   int fmt_down, const void *down_blocks, int64_t down_stride_bytes, int n_expert,
                   const int32_t *expert_ids, const float *g, int n_sel, int64_t hidden, int64_t inter,
                   const float *x, float *y, qmv_stream_t stream)
{
    if (!gate_blocks || !up_blocks || !down_blocks || !expert_ids || !g || !x || !y) return QMV_ERR_NULL;
    if (n_sel >= 1 && inter >= 1 && (int64_t)n_sel * inter > QMV_STATIC_H_FLOATS) return QMV_ERR_SHAPE;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        (void)cudaGetLastError();
        return QMV_ERR_DEVICE;
    }
    float *h = nullptr;
    {
        // once per device, with that device current: the array's device address
        // (its name in host code is only a host-side stand-in)
        std::lock_guard<std::mutex> lk(g_mu);
        if (!g_dev[dev].static_h) {
            void *ptr = nullptr;
            const cudaError_t e = cudaGetSymbolAddress(&ptr, g_static_h);
            if (e != cudaSuccess) return cuda_fail(e);
            g_dev[dev].static_h = static_cast<float *>(ptr);
        }
        h = g_dev[dev].static_h;
    }
    return moe_ffn(fmt_gu, gate_blocks, up_blocks, gu_stride_bytes, fmt_down, down_blocks, down_stride_bytes,
                   n_expert, expert_ids, g, n_sel, hidden, inter, x, h, y, stream);
}

int qmv_argmax_ws(int fmt, const void *W_blocks, int64_t rows, int64_t cols, const float *x, float *y, int n_tok,
                  int32_t *idx_out, void *workspace, qmv_stream_t stream)
{
    int rc = argmax_check(fmt, W_blocks, rows, cols, x, y, n_tok, idx_out);
    if (rc) return rc;
    if (!workspace) return QMV_ERR_NULL;
    if (!aligned(workspace, 8)) return QMV_ERR_ALIGN;
    DevInfo di;
    if ((rc = get_dev(di))) return rc;
    unsigned long long *keys = static_cast<unsigned long long *>(workspace);
    unsigned *done = reinterpret_cast<unsigned *>(keys + QMV_MAX_NTOK);
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (n_tok == 1) {
        // one launch: the streaming kernel folds each CTA's best row into the key
        const SkGeom g = sk_geom(fmt, SK_PLAIN, rows, cols, 1, 0, 1, di.sm_count);
        if (g.ok && g.ksegs == 1) {
            if (injected_failure()) return QMV_ERR_CUDA;
            return sk_single(fmt, W_blocks, rows, cols, x, y, g, di, st, idx_out, keys, done);
        }
    }
    if ((rc = qmv_batched(fmt, W_blocks, rows, cols, x, y, n_tok, stream))) return rc;
    const dim3 grid((unsigned)ceil_div(rows, ARGMAX_ROWS_PER_CTA), (unsigned)n_tok);
    argmax_rows_kernel<<<grid, ARGMAX_THREADS, 0, st>>>(y, rows, rows, idx_out, keys, done);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e);
    return QMV_OK;
}

int qmv_argmax(int fmt, const void *W_blocks, int64_t rows, int64_t cols, const float *x, float *y, int n_tok,
               int32_t *idx_out, qmv_stream_t stream)
{
    int rc = argmax_check(fmt, W_blocks, rows, cols, x, y, n_tok, idx_out);
    if (rc) return rc;
    DevInfo di;
    if ((rc = get_dev(di))) return rc;
    return qmv_argmax_ws(fmt, W_blocks, rows, cols, x, y, n_tok, idx_out, di.amax_key, stream);
}

int qmv_dequant(int fmt, const void *W_blocks, int64_t rows, int64_t cols, float *out, qmv_stream_t stream)
{
    if (!W_blocks || !out) return QMV_ERR_NULL;
    int rc = check_matrix(fmt, rows, cols);
    if (rc) return rc;
    if (!aligned(W_blocks, 16) || !aligned(out, 4)) return QMV_ERR_ALIGN;
    if (injected_failure()) return QMV_ERR_CUDA;
    DevInfo di;
    if ((rc = get_dev(di))) return rc;
    const int64_t bpr = cols / block_weights(fmt);
    const int64_t nblk = rows * bpr;
    const unsigned grid = (unsigned)std::min<int64_t>(ceil_div(nblk, 256), (int64_t)di.sm_count * 16);
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const uint8_t *W = static_cast<const uint8_t *>(W_blocks);
    by_fmt(fmt, [&](auto f) { dequant_kernel<decltype(f)::value><<<grid, 256, 0, st>>>(W, nblk, bpr, cols, out); });
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e);
    return QMV_OK;
}

int qmv_check(qmv_stream_t stream, int *dev_err_out)
{
    if (dev_err_out) *dev_err_out = 0;
    const cudaError_t se = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
    if (se != cudaSuccess) return cuda_fail(se);
    DevInfo di;
    int rc = get_dev(di);
    if (rc) return rc;
    int word = 0;
    if (cudaMemcpy(&word, di.err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemset(di.err, 0, sizeof(int)) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) {
        (void)cudaGetLastError();
        return QMV_ERR_CUDA;
    }
    if (word && (cudaMemset(di.amax_key, 0, QMV_ARGMAX_WS_BYTES) != cudaSuccess ||
                 cudaDeviceSynchronize() != cudaSuccess)) {
        (void)cudaGetLastError();
        return QMV_ERR_CUDA;
    }
    if (dev_err_out) *dev_err_out = word;
    return word ? QMV_ERR_DEVICE : QMV_OK;
}

}  // extern "C"
