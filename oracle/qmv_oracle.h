/*
 * qmv_oracle.h -- the oracle: a plain, slow CPU restatement of the quantized
 * decode-step matvec, used ONLY as test infrastructure (tests, the smoke check
 * and the CPU-baseline leg of the benchmark).  No product code links it, and it
 * shares no source, header, table or helper with the CUDA library.
 *
 * What it computes, and where that is stated:
 *   - GGUF block formats Q8_0 / Q4_K / Q6_K (and Q4_0 / Q5_K, named among the
 *     formats FlareLLM supports), dequantized at run time to f32, activations
 *     kept in f32:
 *       BebeLM：纯Rust实现的端侧大模型推理引擎, §量化格式支持 (Q4_K: 256
 *       weights per superblock in 144 bytes; Q6_K for sensitive tensors;
 *       dequantization at run time, f32 activations);
 *       FlareLLM：纯Rust打造的浏览器端LLM推理引擎, §量化技术的全面支持 and
 *       §计算路径的智能选择 (Q8_0, K-quants), §生态对比与定位 (standard GGUF);
 *       Wick：纯Rust编写的高性能LLM推理引擎, §量化支持 (Q4_K_M, Q8_0).
 *     The pages give no bit layout beyond the Q4_K size; the GGUF on-disk
 *     layout is the reading adopted (spelled out at each decoder below).
 *   - y = W x for 1..8 tokens (FlareLLM page, §推理层面的深度优化: fused QKV /
 *     gate-up projections and n-gram speculative decoding, i.e. several tokens
 *     verified against one pass over the weights).
 *   - MoE router and expert FFN: BebeLM page, §核心算子 (MoE前馈网络: sigmoid
 *     router, top-4 of 32 experts, expert bias for selection only, normalised
 *     weights norm_topk_prob) and §混合专家（MoE）架构.
 *
 * Parity status of each function is recorded beside it ("pinned by ...").
 * Build: plain C99, -O2 -ffp-contract=off (no FMA contraction), optional OpenMP.
 */
#ifndef QMV_ORACLE_H
#define QMV_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORC_Q8_0 = 0, ORC_Q4_K = 1, ORC_Q6_K = 2, ORC_Q4_0 = 3, ORC_Q5_K = 4 };

/* IEEE binary16 bit pattern -> f32, decoded bit by bit (exact). */
float orc_half_to_float(uint16_t h);

/* Weights per block (32, 256, 256) and bytes per block (34, 144, 210); 0 for
 * an unknown format. */
int orc_block_weights(int fmt);
int orc_block_bytes(int fmt);

/* Dequantize one block into f32 weights (32 or 256 values). */
void orc_dequant_block_q8_0(const uint8_t *blk, float *w);
void orc_dequant_block_q4_k(const uint8_t *blk, float *w);
void orc_dequant_block_q6_k(const uint8_t *blk, float *w);
void orc_dequant_block_q4_0(const uint8_t *blk, float *w);
void orc_dequant_block_q5_k(const uint8_t *blk, float *w);

/* Dequantize a dense row-major matrix of rows x cols weights (row r starts at
 * byte r * (cols / block_weights) * block_bytes) into out[rows][cols].
 * Returns 0, or -1 for a bad format / shape. */
int orc_dequant(int fmt, const uint8_t *W, int64_t rows, int64_t cols, float *out);

/* y[t][r] = sum_i (double)w[r][i] * (double)x[t][i], summed in f64 in index
 * order; bound[t][r] = sum_i |w[r][i] * x[t][i]| in f64.  x is [n_tok][cols],
 * y and bound are [n_tok][rows] (either output may be NULL).  nthreads > 1
 * splits rows over OpenMP threads when built with OpenMP (the arithmetic of a
 * row does not change).  Returns 0 or -1. */
int orc_qmv(int fmt, const uint8_t *W, int64_t rows, int64_t cols,
            const float *x, int n_tok, double *y, double *bound, int nthreads);

/* Same as orc_qmv for the listed rows only: y and bound are [n_tok][n_rows],
 * entry (t, k) belongs to row row_idx[k]. */
int orc_qmv_rows(int fmt, const uint8_t *W, int64_t rows, int64_t cols,
                 const int64_t *row_idx, int64_t n_rows,
                 const float *x, int n_tok, double *y, double *bound);

/* MoE router (BebeLM page, §核心算子, MoE前馈网络).  In f32, the precision of
 * the device router, since the result is a discrete choice:
 *   s_e = 1 / (1 + exp(-logit_e)),   b_e = s_e + bias_e (selection only).
 * Picks the top_k experts by b (ties to the lower index), in descending b,
 * writes their ids, and the weights g_k = s_{id_k} / sum_j s_{id_j} computed in
 * f64 from the f64 sigmoid.  biased_out[n_expert] (may be NULL) receives b.
 * Returns 0, or -1 for bad sizes. */
int orc_route(const float *logits, const float *bias, int n_expert, int top_k,
              int32_t *ids, double *g, float *biased_out);

/* silu(z) = z / (1 + exp(-z)) in f64. */
double orc_silu(double z);

/* One MoE FFN step for n_sel selected experts, all in f64 from the exact f32
 * dequantized weights (BebeLM page, §核心算子: experts are SwiGLU FFNs whose
 * outputs are combined with the normalised router weights):
 *   u_k = G_{id_k} x,  v_k = U_{id_k} x,  h_k = silu(u_k) * v_k,
 *   y   = sum_k g_k * D_{id_k} h_k.
 * Expert e's gate / up matrix is [inter x hidden] at gate_base + e*gu_stride
 * (resp. up_base); its down matrix is [hidden x inter] at
 * down_base + e*down_stride.  Outputs (each may be NULL): u, v, h as
 * [n_sel][inter], y as [hidden].  Returns 0 or -1. */
int orc_moe_ffn(int fmt_gu, const uint8_t *gate_base, const uint8_t *up_base,
                int64_t gu_stride, int fmt_down, const uint8_t *down_base,
                int64_t down_stride, int n_expert, const int32_t *ids,
                const double *g, int n_sel, int64_t hidden, int64_t inter,
                const float *x, double *u, double *v, double *h, double *y);

#ifdef __cplusplus
}
#endif
#endif
