// qmv_dispatch.cuh -- runtime (n_tok, R, x-in-registers) -> kernel instance,
// instantiated once per format by qmv_fmt_*.cu so the three formats compile in
// parallel.
#pragma once

#include "qmv_kernels.cuh"

namespace qmv {

template <int FMT, int NTOK, int R, bool XREG>
static cudaError_t launch_one(const Params &p, dim3 grid, size_t smem, cudaStream_t stream, bool pdl)
{
    auto kern = qmv_pipeline_kernel<FMT, NTOK, R, XREG>;
    // Raise the dynamic shared-memory limit once per (kernel, device).
    static int configured[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (configured[dev] < (int)smem) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        configured[dev] = (int)smem;
    }
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(NTHREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = pdl ? attr : nullptr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, p);
}

template <int FMT, int NTOK>
static cudaError_t launch_ntok(const Params &p, const KernelChoice &kc, dim3 grid, size_t smem,
                               cudaStream_t stream)
{
    if (kc.xreg) {
        if constexpr (NTOK == 1) {
            switch (kc.R) {
            case 1: return launch_one<FMT, 1, 1, true>(p, grid, smem, stream, kc.pdl);
            case 2: return launch_one<FMT, 1, 2, true>(p, grid, smem, stream, kc.pdl);
            case 4: return launch_one<FMT, 1, 4, true>(p, grid, smem, stream, kc.pdl);
            case 8: return launch_one<FMT, 1, 8, true>(p, grid, smem, stream, kc.pdl);
            default: return cudaErrorInvalidValue;
            }
        }
        return cudaErrorInvalidValue;
    }
    switch (kc.R) {
    case 1: return launch_one<FMT, NTOK, 1, false>(p, grid, smem, stream, kc.pdl);
    case 2: return launch_one<FMT, NTOK, 2, false>(p, grid, smem, stream, kc.pdl);
    case 4: return launch_one<FMT, NTOK, 4, false>(p, grid, smem, stream, kc.pdl);
    case 8:
        if constexpr (NTOK == 1) return launch_one<FMT, NTOK, 8, false>(p, grid, smem, stream, kc.pdl);
        return cudaErrorInvalidValue;
    default: return cudaErrorInvalidValue;
    }
}

template <int FMT>
cudaError_t launch_pipeline(const Params &p, const KernelChoice &kc, dim3 grid, size_t smem,
                            cudaStream_t stream)
{
    switch (kc.ntok) {
    case 1: return launch_ntok<FMT, 1>(p, kc, grid, smem, stream);
    case 2: return launch_ntok<FMT, 2>(p, kc, grid, smem, stream);
    case 3: return launch_ntok<FMT, 3>(p, kc, grid, smem, stream);
    case 4: return launch_ntok<FMT, 4>(p, kc, grid, smem, stream);
    case 5: return launch_ntok<FMT, 5>(p, kc, grid, smem, stream);
    case 6: return launch_ntok<FMT, 6>(p, kc, grid, smem, stream);
    case 7: return launch_ntok<FMT, 7>(p, kc, grid, smem, stream);
    case 8: return launch_ntok<FMT, 8>(p, kc, grid, smem, stream);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace qmv
