// Kernel instances of the quantized matvec for one block format.  This format
// runs on the general pipeline and the streaming kernels only (the warp-ring
// and tensor-core kernels are built for Q8_0, Q4_K and Q6_K).
#include "qmv_dispatch.cuh"

namespace qmv {
template cudaError_t launch_pipeline<FMT_Q4_0>(const Params &, const KernelChoice &, dim3, size_t, cudaStream_t);
template cudaError_t launch_multi<FMT_Q4_0>(const MultiParams &, const KernelChoice &, int, size_t, cudaStream_t);
template cudaError_t launch_sk<FMT_Q4_0>(const SkParams &, int, int, dim3, size_t, cudaStream_t, bool);
template cudaError_t launch_skt<FMT_Q4_0>(const SkParams &, int, int, dim3, size_t, cudaStream_t, bool);
template cudaError_t launch_skm<FMT_Q4_0>(const SkMoeParams &, int, dim3, size_t, cudaStream_t);
}  // namespace qmv
