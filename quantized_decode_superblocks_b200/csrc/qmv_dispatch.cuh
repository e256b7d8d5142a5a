// qmv_dispatch.cuh -- runtime (n_tok, R, x-in-registers) -> kernel instance,
// instantiated once per format by qmv_fmt_*.cu so the formats compile in
// parallel.
#pragma once

#include <atomic>
#include <mutex>

#include "qmv_rw.cuh"
#include "qmv_sk.cuh"
#include "qmv_skt.cuh"
#include "qmv_tc.cuh"

namespace qmv {

// Per (kernel, device): the dynamic shared-memory limit set so far.
using SmemCfg = std::atomic<int>[64];

// Raises kern's dynamic shared-memory limit on the current device to at least
// smem.  Host threads may race here: the fast path is one atomic load, and the
// raise itself runs under a lock so the limit only ever grows.
template <class Kern>
static cudaError_t ensure_smem(Kern kern, SmemCfg &configured, size_t smem)
{
    static std::mutex mu;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (configured[dev].load(std::memory_order_acquire) >= (int)smem) return cudaSuccess;
    std::lock_guard<std::mutex> lk(mu);
    if (configured[dev].load(std::memory_order_relaxed) >= (int)smem) return cudaSuccess;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured[dev].store((int)smem, std::memory_order_release);
    return cudaSuccess;
}

// Launch `kern` with `arg`: raises the dynamic shared-memory limit once per
// (kernel, device) and adds the programmatic-serialization attribute when asked.
template <class Kern, class Arg>
static cudaError_t launch_with(Kern kern, SmemCfg &configured, const Arg &arg, dim3 grid, size_t smem,
                               cudaStream_t stream, bool pdl, bool cooperative = false, int threads = NTHREADS)
{
    cudaError_t e = ensure_smem(kern, configured, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchAttribute attr[2];
    unsigned n_attr = 0;
    if (pdl) {
        attr[n_attr].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n_attr].val.programmaticStreamSerializationAllowed = 1;
        ++n_attr;
    }
    if (cooperative) {      // all CTAs co-resident, or the launch fails (grid barriers)
        attr[n_attr].id = cudaLaunchAttributeCooperative;
        attr[n_attr].val.cooperative = 1;
        ++n_attr;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = n_attr ? attr : nullptr;
    cfg.numAttrs = n_attr;
    return cudaLaunchKernelEx(&cfg, kern, arg);
}

template <int FMT, int NTOK, int R, bool XREG>
struct Instance {
    static cudaError_t one(const Params &p, dim3 grid, size_t smem, cudaStream_t st, bool pdl)
    {
        static SmemCfg configured;
        return launch_with(qmv_pipeline_kernel<FMT, NTOK, R, XREG>, configured, p, grid, smem, st, pdl);
    }
    static cudaError_t multi(const MultiParams &mp, dim3 grid, size_t smem, cudaStream_t st, bool pdl)
    {
        static SmemCfg configured;
        return launch_with(qmv_multi_kernel<FMT, NTOK, R, XREG>, configured, mp, grid, smem, st, pdl);
    }
};

// Calls Fn::template run<FMT, NTOK, R, XREG>() for the runtime choice.
template <int FMT, int NTOK, class Fn>
static cudaError_t pick_r(const KernelChoice &kc, Fn &&fn)
{
    if (kc.xreg) {
        if constexpr (NTOK == 1) {
            switch (kc.R) {
            case 1: return fn.template run<FMT, 1, 1, true>();
            case 2: return fn.template run<FMT, 1, 2, true>();
            case 4: return fn.template run<FMT, 1, 4, true>();
            case 8: return fn.template run<FMT, 1, 8, true>();
            default: return cudaErrorInvalidValue;
            }
        }
        return cudaErrorInvalidValue;
    }
    switch (kc.R) {
    case 1: return fn.template run<FMT, NTOK, 1, false>();
    case 2: return fn.template run<FMT, NTOK, 2, false>();
    case 4: return fn.template run<FMT, NTOK, 4, false>();
    case 8:
        if constexpr (NTOK == 1) return fn.template run<FMT, NTOK, 8, false>();
        return cudaErrorInvalidValue;
    default: return cudaErrorInvalidValue;
    }
}

template <int FMT, class Fn>
static cudaError_t pick(const KernelChoice &kc, Fn &&fn)
{
    switch (kc.ntok) {
    case 1: return pick_r<FMT, 1>(kc, fn);
    case 2: return pick_r<FMT, 2>(kc, fn);
    case 3: return pick_r<FMT, 3>(kc, fn);
    case 4: return pick_r<FMT, 4>(kc, fn);
    case 5: return pick_r<FMT, 5>(kc, fn);
    case 6: return pick_r<FMT, 6>(kc, fn);
    case 7: return pick_r<FMT, 7>(kc, fn);
    case 8: return pick_r<FMT, 8>(kc, fn);
    default: return cudaErrorInvalidValue;
    }
}

struct OneLaunch {
    const Params &p;
    dim3 grid;
    size_t smem;
    cudaStream_t st;
    bool pdl;
    template <int FMT, int NTOK, int R, bool XREG>
    cudaError_t run() const { return Instance<FMT, NTOK, R, XREG>::one(p, grid, smem, st, pdl); }
};

struct MultiLaunch {
    const MultiParams &mp;
    dim3 grid;
    size_t smem;
    cudaStream_t st;
    bool pdl;
    template <int FMT, int NTOK, int R, bool XREG>
    cudaError_t run() const { return Instance<FMT, NTOK, R, XREG>::multi(mp, grid, smem, st, pdl); }
};

template <int FMT, int R, int NT, int NTOK = 1>
struct RwInstance {
    static SmemCfg &configured()
    {
        static SmemCfg c;
        return c;
    }
    static cudaError_t go(const RwParamsT<NT> &p, dim3 grid, size_t smem, cudaStream_t st, bool pdl, bool coop)
    {
        return launch_with(qmv_rw_kernel<FMT, R, NT, NTOK>, configured(), p, grid, smem, st, pdl, coop);
    }
};

template <int FMT, int NT>
cudaError_t launch_rw(const RwParamsT<NT> &p, int R, dim3 grid, size_t smem, cudaStream_t stream, bool pdl,
                      bool cooperative)
{
    switch (R) {
    case 1: return RwInstance<FMT, 1, NT>::go(p, grid, smem, stream, pdl, cooperative);
    case 2: return RwInstance<FMT, 2, NT>::go(p, grid, smem, stream, pdl, cooperative);
    case 4: return RwInstance<FMT, 4, NT>::go(p, grid, smem, stream, pdl, cooperative);
    default: return cudaErrorInvalidValue;
    }
}

template <int FMT, int NTOK>
static cudaError_t launch_rw_mt_r(const RwParams1 &p, int R, dim3 grid, size_t smem, cudaStream_t stream, bool pdl)
{
    switch (R) {
    case 1: return RwInstance<FMT, 1, 1, NTOK>::go(p, grid, smem, stream, pdl, false);
    case 2: return RwInstance<FMT, 2, 1, NTOK>::go(p, grid, smem, stream, pdl, false);
    default: return cudaErrorInvalidValue;
    }
}

template <int FMT>
cudaError_t launch_rw_mt(const RwParams1 &p, int n_tok, int R, dim3 grid, size_t smem, cudaStream_t stream, bool pdl)
{
    switch (n_tok) {
    case 2: return launch_rw_mt_r<FMT, 2>(p, R, grid, smem, stream, pdl);
    case 3: return launch_rw_mt_r<FMT, 3>(p, R, grid, smem, stream, pdl);
    case 4: return launch_rw_mt_r<FMT, 4>(p, R, grid, smem, stream, pdl);
    default: return cudaErrorInvalidValue;      // 5..8 tokens take the general kernel
    }
}

template <int FMT>
cudaError_t launch_pipeline(const Params &p, const KernelChoice &kc, dim3 grid, size_t smem,
                            cudaStream_t stream)
{
    return pick<FMT>(kc, OneLaunch{p, grid, smem, stream, kc.pdl});
}

template <int FMT>
cudaError_t launch_multi(const MultiParams &mp, const KernelChoice &kc, int grid, size_t smem,
                         cudaStream_t stream)
{
    return pick<FMT>(kc, MultiLaunch{mp, dim3((unsigned)grid), smem, stream, kc.pdl});
}

// The one-token streaming kernel: form (plain, SwiGLU, gathered experts) and
// rows per consumer warp.
template <int FMT, int MODE>
static cudaError_t launch_sk_mode(const SkParams &p, int R, dim3 grid, size_t smem, cudaStream_t st, bool pdl)
{
    static SmemCfg c1, c2, c4;
    switch (R) {
    case 1: return launch_with(qmv_sk_kernel<FMT, 1, MODE>, c1, p, grid, smem, st, pdl, false, SK_THREADS);
    case 2: return launch_with(qmv_sk_kernel<FMT, 2, MODE>, c2, p, grid, smem, st, pdl, false, SK_THREADS);
    case 4:
        if constexpr (MODE == SK_PLAIN)
            return launch_with(qmv_sk_kernel<FMT, 4, MODE>, c4, p, grid, smem, st, pdl, false, SK_THREADS);
        return cudaErrorInvalidValue;
    default: return cudaErrorInvalidValue;
    }
}

template <int FMT>
cudaError_t launch_sk(const SkParams &p, int mode, int R, dim3 grid, size_t smem, cudaStream_t st, bool pdl)
{
    switch (mode) {
    case SK_PLAIN: return launch_sk_mode<FMT, SK_PLAIN>(p, R, grid, smem, st, pdl);
    case SK_SWIGLU: return launch_sk_mode<FMT, SK_SWIGLU>(p, R, grid, smem, st, pdl);
    case SK_GATHER: return launch_sk_mode<FMT, SK_GATHER>(p, R, grid, smem, st, pdl);
    default: return cudaErrorInvalidValue;
    }
}

// The streaming kernel's several-token form (plain matrices).
template <int FMT, int NTOK>
static cudaError_t launch_skt_r(const SkParams &p, int R, dim3 grid, size_t smem, cudaStream_t st, bool pdl)
{
    static SmemCfg c1, c2, c4;
    switch (R) {
    case 1: return launch_with(qmv_skt_kernel<FMT, 1, NTOK>, c1, p, grid, smem, st, pdl, false, SK_THREADS);
    case 2: return launch_with(qmv_skt_kernel<FMT, 2, NTOK>, c2, p, grid, smem, st, pdl, false, SK_THREADS);
    case 4:
        if constexpr (NTOK == 2)
            return launch_with(qmv_skt_kernel<FMT, 4, NTOK>, c4, p, grid, smem, st, pdl, false, SK_THREADS);
        return cudaErrorInvalidValue;
    default: return cudaErrorInvalidValue;
    }
}

template <int FMT>
cudaError_t launch_skt(const SkParams &p, int n_tok, int R, dim3 grid, size_t smem, cudaStream_t st, bool pdl)
{
    switch (n_tok) {
    case 2: return launch_skt_r<FMT, 2>(p, R, grid, smem, st, pdl);
    case 3: return launch_skt_r<FMT, 3>(p, R, grid, smem, st, pdl);
    case 4: return launch_skt_r<FMT, 4>(p, R, grid, smem, st, pdl);
    default: return cudaErrorInvalidValue;
    }
}

// The one-launch MoE FFN step (cooperative: one CTA per SM, all resident).
template <int FMT>
cudaError_t launch_skm(const SkMoeParams &p, int R, dim3 grid, size_t smem, cudaStream_t st)
{
    static SmemCfg c1, c2;
    switch (R) {
    case 1: return launch_with(qmv_skm_kernel<FMT, 1>, c1, p, grid, smem, st, false, true, SK_THREADS);
    case 2: return launch_with(qmv_skm_kernel<FMT, 2>, c2, p, grid, smem, st, false, true, SK_THREADS);
    default: return cudaErrorInvalidValue;
    }
}

// The tensor-core several-token kernel (Q8_0): x in shared memory or through L2.
template <int FMT>
cudaError_t launch_tc(const TcParams &p, bool x_smem, dim3 grid, size_t smem, cudaStream_t st, bool pdl)
{
    static SmemCfg configured_s, configured_g;
    if constexpr (FMT == FMT_Q6_K) {       // x always in shared memory
        if (!x_smem) return cudaErrorInvalidValue;
        return launch_with(qmv_tc_kernel<FMT, TC_WARPS, true>, configured_s, p, grid, smem, st, pdl, false, TC_WARPS * 32);
    } else {
        if (x_smem)
            return launch_with(qmv_tc_kernel<FMT, TC_WARPS, true>, configured_s, p, grid, smem, st, pdl, false,
                               TC_WARPS * 32);
        return launch_with(qmv_tc_kernel<FMT, TC_WARPS, false>, configured_g, p, grid, smem, st, pdl, false,
                           TC_WARPS * 32);
    }
}

}  // namespace qmv
