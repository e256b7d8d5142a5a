// qmv_misc.cuh -- the MoE router kernel and the dequant-only kernel (one
// translation unit: qmv_api.cu).
#pragma once

#include "qmv_kernels.cuh"

namespace qmv {

// ------------------------------------------------------- greedy argmax --
// FlareLLM page, §推理层面的深度优化 (greedy decoding picks the next token from
// the logits on the device): idx[t] = the row of the largest y[t][row] (IEEE >
// on f32), ties to the lower row, NaN skipped; -1 when every value is NaN.
// A grid of CTAs per token scans the rows (float4 loads from L2, where the
// projection just wrote them); each CTA folds its best (value, row) into one
// 64-bit key per token with atomicMax -- the value's bits mapped to an
// order-preserving unsigned in the high word, the complement of the row in the
// low word, so a larger key is a larger value or, for equal values, a lower
// row: the result does not depend on the order of the atomics.  The last CTA
// of the token (an arrival counter) writes idx and puts the key and the
// counter back to zero for the next call.
constexpr int ARGMAX_THREADS = 256;
constexpr int ARGMAX_ROWS_PER_CTA = 2048;

__global__ void __launch_bounds__(ARGMAX_THREADS) argmax_rows_kernel(const float *y, int64_t rows,
                                                                     int64_t y_tok_stride, int32_t *idx,
                                                                     unsigned long long *keys, unsigned *done)
{
    __shared__ float s_v[ARGMAX_THREADS / 32];
    __shared__ int s_i[ARGMAX_THREADS / 32];
    const int t = (int)blockIdx.y;
    const float *yt = y + (int64_t)t * y_tok_stride;
    const int64_t r0 = (int64_t)blockIdx.x * ARGMAX_ROWS_PER_CTA;
    const int64_t r1 = min(rows, r0 + ARGMAX_ROWS_PER_CTA);
    float bv = 0.f;
    int bi = -1;
    const bool vec = ((reinterpret_cast<uintptr_t>(yt + r0) & 15u) == 0);
    const int64_t n4 = vec ? (r1 - r0) / 4 : 0;
    for (int64_t i = threadIdx.x; i < n4; i += ARGMAX_THREADS) {
        const float4 v = __ldcg(reinterpret_cast<const float4 *>(yt + r0) + i);
        const float e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int k = 0; k < 4; ++k)
            if (e[k] == e[k]) argmax_merge(bv, bi, e[k], (int)(r0 + 4 * i + k));
    }
    for (int64_t r = r0 + 4 * n4 + threadIdx.x; r < r1; r += ARGMAX_THREADS) {
        const float e = __ldcg(yt + r);
        if (e == e) argmax_merge(bv, bi, e, (int)r);
    }
    for (int o = 16; o >= 1; o >>= 1)
        argmax_merge(bv, bi, __shfl_xor_sync(0xFFFFFFFFu, bv, o), __shfl_xor_sync(0xFFFFFFFFu, bi, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) {
        s_v[warp] = bv;
        s_i[warp] = bi;
    }
    __syncthreads();
    if (warp == 0) {
        bv = lane < ARGMAX_THREADS / 32 ? s_v[lane] : 0.f;
        bi = lane < ARGMAX_THREADS / 32 ? s_i[lane] : -1;
        for (int o = 16; o >= 1; o >>= 1)
            argmax_merge(bv, bi, __shfl_xor_sync(0xFFFFFFFFu, bv, o), __shfl_xor_sync(0xFFFFFFFFu, bi, o));
        if (lane == 0) {
            if (bi >= 0) atomicMax(keys + t, argmax_key(bv, bi));
            __threadfence();
            if (atomicAdd(done + t, 1u) == gridDim.x - 1u) {      // the token's last CTA
                __threadfence();
                const unsigned long long k = atomicExch(keys + t, 0ull);
                atomicExch(done + t, 0u);
                idx[t] = k ? (int32_t)(0xFFFFFFFFu - (uint32_t)(k & 0xFFFFFFFFull)) : -1;
            }
        }
    }
}

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
        else if (FMT == FMT_Q4_0) dequant_block_q4_0(blk, o);
        else if (FMT == FMT_Q4_K) dequant_block_q4_k(blk, o);
        else if (FMT == FMT_Q5_K) dequant_block_q5_k(blk, o);
        else dequant_block_q6_k(blk, o);
    }
}

}  // namespace qmv
