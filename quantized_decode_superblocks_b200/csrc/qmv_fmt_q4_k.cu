// Kernel instances of the quantized matvec pipeline for one block format.
#include "qmv_dispatch.cuh"

namespace qmv {
template cudaError_t launch_pipeline<FMT_Q4_K>(const Params &, const KernelChoice &, dim3, size_t, cudaStream_t);
template cudaError_t launch_multi<FMT_Q4_K>(const MultiParams &, const KernelChoice &, int, size_t, cudaStream_t);
template cudaError_t launch_rw<FMT_Q4_K, 1>(const RwParams1 &, int, dim3, size_t, cudaStream_t, bool, bool);
template cudaError_t launch_rw_mt<FMT_Q4_K>(const RwParams1 &, int, int, dim3, size_t, cudaStream_t, bool);
template cudaError_t launch_tc<FMT_Q4_K>(const TcParams &, bool, dim3, size_t, cudaStream_t, bool);
template cudaError_t launch_sk<FMT_Q4_K>(const SkParams &, int, int, dim3, size_t, cudaStream_t, bool);
template cudaError_t launch_skt<FMT_Q4_K>(const SkParams &, int, int, dim3, size_t, cudaStream_t, bool);
template cudaError_t launch_skm<FMT_Q4_K>(const SkMoeParams &, int, dim3, size_t, cudaStream_t);
}  // namespace qmv
