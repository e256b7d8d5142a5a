// qmv_misc.cuh -- the MoE router kernel and the dequant-only kernel (one
// translation unit: qmv_api.cu).
#pragma once

#include "qmv_kernels.cuh"

namespace qmv {

// -------------------------------------------------------------- router --
// BebeLM page, §核心算子 (MoE前馈网络): sigmoid scores, the per-expert bias
// added for the choice only, top_k by biased score (ties to the lower index),
// weights normalised over the chosen unbiased scores.  One warp.
__global__ void __launch_bounds__(32) moe_route_kernel(const float *logits, const float *bias,
                                                       int n_expert, int top_k,
                                                       int32_t *ids, float *g)
{
    __shared__ float s_score[1024];
    __shared__ float s_biased[1024];
    __shared__ unsigned char s_taken[1024];
    __shared__ float s_sel[8];
    const int lane = threadIdx.x;
    for (int e = lane; e < n_expert; e += 32) {
        const float s = 1.0f / (1.0f + expf(-logits[e]));
        s_score[e] = s;
        s_biased[e] = s + bias[e];
        s_taken[e] = 0;
    }
    __syncwarp();
    for (int k = 0; k < top_k; ++k) {
        float bv = 0.f;
        int bi = -1;
        for (int e = lane; e < n_expert; e += 32) {
            if (s_taken[e]) continue;
            const float v = s_biased[e];
            if (bi < 0 || v > bv) { bv = v; bi = e; }   // ascending e: ties keep the lower index
        }
        for (int o = 16; o >= 1; o >>= 1) {
            const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, o);
            const int oi = __shfl_xor_sync(0xFFFFFFFFu, bi, o);
            const bool better = (oi >= 0) && (bi < 0 || ov > bv || (ov == bv && oi < bi));
            if (better) { bv = ov; bi = oi; }
        }
        if (lane == 0) {
            ids[k] = bi;
            s_taken[bi] = 1;
            s_sel[k] = s_score[bi];
        }
        __syncwarp();
    }
    if (lane == 0) {
        float total = 0.f;
        for (int k = 0; k < top_k; ++k) total += s_sel[k];
        for (int k = 0; k < top_k; ++k) g[k] = s_sel[k] / total;
    }
}

// ------------------------------------------------------- dequant-only --
template <int FMT>
__global__ void __launch_bounds__(256) dequant_kernel(const uint8_t *W, int64_t n_blocks,
                                                      int64_t blocks_per_row, int64_t cols, float *out)
{
    constexpr int BW = Fmt<FMT>::BW, BB = Fmt<FMT>::BB;
    for (int64_t bi = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; bi < n_blocks;
         bi += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = bi / blocks_per_row, b = bi % blocks_per_row;
        float *o = out + r * cols + b * BW;
        const uint8_t *blk = W + bi * BB;
        if (FMT == FMT_Q8_0) dequant_block_q8_0(blk, o);
        else if (FMT == FMT_Q4_K) dequant_block_q4_k(blk, o);
        else dequant_block_q6_k(blk, o);
    }
}

}  // namespace qmv
