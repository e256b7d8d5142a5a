// Kernel instances of the quantized matvec pipeline for one block format.
#include "qmv_dispatch.cuh"

namespace qmv {
template cudaError_t launch_pipeline<FMT_Q4_K>(const Params &, const KernelChoice &, dim3, size_t, cudaStream_t);
template cudaError_t launch_multi<FMT_Q4_K>(const MultiParams &, const KernelChoice &, int, size_t, cudaStream_t);
}  // namespace qmv
