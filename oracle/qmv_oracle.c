/*
 * qmv_oracle.c -- the oracle (test infrastructure only; see qmv_oracle.h).
 *
 * Plain C, f64 accumulation, no blocking, no fusion, no reordering beyond the
 * definitions below.  Built with -ffp-contract=off so that every f32 product
 * and sum is rounded exactly as written.
 *
 * Sources of each definition (page title, section):
 *   [BebeLM]  BebeLM：纯Rust实现的端侧大模型推理引擎
 *             §量化格式支持 -- Q4_K superblock of 256 weights in 144 bytes, Q6_K
 *             for sensitive tensors, run-time dequantization, f32 activations;
 *             §核心算子 (MoE前馈网络) -- sigmoid router, top-k = 4 of 32 experts,
 *             expert bias used for selection only, normalised weights.
 *   [Flare]   FlareLLM：纯Rust打造的浏览器端LLM推理引擎
 *             §量化技术的全面支持 / §计算路径的智能选择 -- Q8_0, K-quants;
 *             §生态对比与定位 -- standard GGUF;
 *             §推理层面的深度优化 -- fused QKV / gate-up matvecs, speculative
 *             multi-token verification.
 *   [Wick]    Wick：纯Rust编写的高性能LLM推理引擎, §量化支持 -- Q4_K_M, Q8_0.
 * The pages fix only the Q4_K size; the byte layout of each block is the GGUF
 * on-disk layout (the engines claim standard GGUF), restated at each decoder.
 */
#include "qmv_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------- fp16 -- */

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.
 * Normal:    (-1)^s * (1024 + f) * 2^(e - 25)
 * Subnormal: (-1)^s * f * 2^-24
 * e == 31:   infinity (f == 0) or NaN.
 * Every binary16 value is exactly representable in f32; ldexp is exact here.
 * Pinned by: all 65536 patterns against numpy's float16 -> float32 cast. */
float orc_half_to_float(uint16_t h)
{
    int s = (h >> 15) & 1;
    int e = (h >> 10) & 31;
    int f = h & 1023;
    double v;
    if (e == 0) {
        v = ldexp((double)f, -24);
    } else if (e == 31) {
        v = (f == 0) ? INFINITY : NAN;
    } else {
        v = ldexp((double)(1024 + f), e - 25);
    }
    return (float)(s ? -v : v);
}

static float half_at(const uint8_t *p)
{
    /* little-endian 16-bit field */
    return orc_half_to_float((uint16_t)(p[0] | (p[1] << 8)));
}

int orc_block_weights(int fmt)
{
    switch (fmt) {
    case ORC_Q8_0: return 32;
    case ORC_Q4_K: return 256;
    case ORC_Q6_K: return 256;
    case ORC_Q4_0: return 32;
    case ORC_Q5_K: return 256;
    default: return 0;
    }
}

int orc_block_bytes(int fmt)
{
    switch (fmt) {
    case ORC_Q8_0: return 2 + 32;            /* d, q[32]                   */
    case ORC_Q4_K: return 2 + 2 + 12 + 128;  /* d, dmin, scales[12], qs[128] */
    case ORC_Q6_K: return 128 + 64 + 16 + 2; /* ql, qh, scales[16], d      */
    case ORC_Q4_0: return 2 + 16;            /* d, qs[16]                  */
    case ORC_Q5_K: return 2 + 2 + 12 + 32 + 128; /* d, dmin, scales[12], qh[32], qs[128] */
    default: return 0;
    }
}

/* ---------------------------------------------------------------- Q8_0 -- */

/* Q8_0 block, 34 bytes: bytes 0-1 fp16 d, bytes 2-33 int8 q[0..31].
 *   w_i = d * q_i          ([Flare] §计算路径的智能选择: Q8_0 int8)
 * d has 11 significant bits and q at most 7, so the product is exact in f32.
 * Pinned by: per-slot round trips through the independent test packer, a
 * second decoder in the tests, hand-worked blocks, closed forms. */
void orc_dequant_block_q8_0(const uint8_t *blk, float *w)
{
    float d = half_at(blk);
    for (int i = 0; i < 32; ++i) {
        int q = (int)(int8_t)blk[2 + i];
        w[i] = d * (float)q;
    }
}

/* ---------------------------------------------------------------- Q4_K -- */

/* Q4_K superblock, 144 bytes ([BebeLM] §量化格式支持: 256 weights in 144 bytes):
 *   bytes 0-1    fp16 d
 *   bytes 2-3    fp16 dmin
 *   bytes 4-15   scales[12]: eight 6-bit sub-block scales sc_j and eight 6-bit
 *                mins m_j, j = 0..7 (one per 32-weight sub-block), packed as
 *                  j < 4 : sc_j = scales[j] & 63,   m_j = scales[j+4] & 63
 *                  j >= 4: sc_j = (scales[j+4] & 15) | ((scales[j-4] >> 6) << 4)
 *                          m_j  = (scales[j+4] >> 4) | ((scales[j]   >> 6) << 4)
 *   bytes 16-143 qs[128]: for chunk c = 0..3 and l = 0..31, byte qs[32c + l]
 *                holds weight 64c + l in its low nibble and weight 64c + 32 + l
 *                in its high nibble.
 * Weight i lies in sub-block j = i / 32 and
 *   w_i = d * sc_j * q_i - dmin * m_j.
 * d*sc_j (17 bits), (d*sc_j)*q_i (21 bits) and dmin*m_j (17 bits) are exact in
 * f32; only the final subtraction rounds (to nearest even).
 * Pinned by: per-slot round trips (every sc/m slot x all 64 values, every
 * nibble position x all 16 values), second decoder, hand-worked blocks,
 * closed forms. */
void orc_dequant_block_q4_k(const uint8_t *blk, float *w)
{
    float d = half_at(blk + 0);
    float dmin = half_at(blk + 2);
    const uint8_t *scales = blk + 4;
    const uint8_t *qs = blk + 16;

    int sc[8], m[8];
    for (int j = 0; j < 8; ++j) {
        if (j < 4) {
            sc[j] = scales[j] & 63;
            m[j] = scales[j + 4] & 63;
        } else {
            sc[j] = (scales[j + 4] & 15) | ((scales[j - 4] >> 6) << 4);
            m[j] = (scales[j + 4] >> 4) | ((scales[j] >> 6) << 4);
        }
    }

    int q[256];
    for (int c = 0; c < 4; ++c) {
        for (int l = 0; l < 32; ++l) {
            uint8_t b = qs[32 * c + l];
            q[64 * c + l] = b & 15;
            q[64 * c + 32 + l] = b >> 4;
        }
    }

    for (int i = 0; i < 256; ++i) {
        int j = i / 32;
        float t1 = d * (float)sc[j];
        float t2 = dmin * (float)m[j];
        w[i] = t1 * (float)q[i] - t2;
    }
}

/* ---------------------------------------------------------------- Q6_K -- */

/* Q6_K superblock, 210 bytes ([BebeLM] §量化格式支持: 6-bit quantization for
 * sensitive tensors):
 *   bytes 0-127   ql[128]: low 4 bits of each 6-bit quant
 *   bytes 128-191 qh[64]:  high 2 bits of each quant
 *   bytes 192-207 scales[16]: int8 scale per 16-weight group
 *   bytes 208-209 fp16 d
 * Write weight i = 128h + 32t + l (h in {0,1}, t in 0..3, l in 0..31):
 *   low  = ql[64h + l + 32*(t & 1)], low nibble if t < 2, high nibble if t >= 2
 *   high = (qh[32h + l] >> (2t)) & 3
 *   q_i  = low | (high << 4)               (0..63)
 *   w_i  = d * scales[i / 16] * (q_i - 32)
 * At most 11 + 6 + 5 significant bits: exact in f32.
 * Pinned by: per-slot round trips (every position x all 64 quants, every
 * scale slot x all 256 int8 values), second decoder, hand-worked blocks,
 * closed forms. */
void orc_dequant_block_q6_k(const uint8_t *blk, float *w)
{
    const uint8_t *ql = blk;
    const uint8_t *qh = blk + 128;
    const int8_t *scales = (const int8_t *)(blk + 192);
    float d = half_at(blk + 208);

    for (int h = 0; h < 2; ++h) {
        for (int t = 0; t < 4; ++t) {
            for (int l = 0; l < 32; ++l) {
                int i = 128 * h + 32 * t + l;
                uint8_t lb = ql[64 * h + l + 32 * (t & 1)];
                int low = (t < 2) ? (lb & 15) : (lb >> 4);
                int high = (qh[32 * h + l] >> (2 * t)) & 3;
                int q = low | (high << 4);
                float ds = d * (float)scales[i / 16];
                w[i] = ds * (float)(q - 32);
            }
        }
    }
}

/* ---------------------------------------------------------------- Q4_0 -- */

/* Q4_0 block, 18 bytes ([Flare] §量化技术的全面支持: the Q4_0 .. Q8_1 family):
 *   bytes 0-1   fp16 d
 *   bytes 2-17  qs[16]: byte qs[j] holds weight j in its low nibble and
 *               weight j + 16 in its high nibble (j = 0..15)
 *   w_i = d * (q_i - 8)                      (q_i = 0..15, so -8..7)
 * 11 + 4 significant bits: exact in f32.
 * Pinned by: per-slot round trips (every position x all 16 values), second
 * decoder, a hand-worked block, closed forms. */
void orc_dequant_block_q4_0(const uint8_t *blk, float *w)
{
    float d = half_at(blk);
    const uint8_t *qs = blk + 2;
    for (int j = 0; j < 16; ++j) {
        int lo = qs[j] & 15;
        int hi = qs[j] >> 4;
        w[j] = d * (float)(lo - 8);
        w[j + 16] = d * (float)(hi - 8);
    }
}

/* ---------------------------------------------------------------- Q5_K -- */

/* Q5_K superblock, 176 bytes ([Flare] §量化技术的全面支持: K-quants Q2K .. Q6K):
 *   bytes 0-1     fp16 d
 *   bytes 2-3     fp16 dmin
 *   bytes 4-15    scales[12]: the eight 6-bit scales sc_j and mins m_j, packed
 *                 exactly as in Q4_K
 *   bytes 16-47   qh[32]: the fifth bit of every quant
 *   bytes 48-175  qs[128]: the low four bits, laid out as the Q4_K nibbles
 * For chunk c = 0..3 and l = 0..31:
 *   weight 64c + l      : low nibble of qs[32c + l], fifth bit = bit 2c   of qh[l]
 *   weight 64c + 32 + l : high nibble of qs[32c + l], fifth bit = bit 2c+1 of qh[l]
 *   q_i = low4 + 16 * bit5                  (0..31)
 * Weight i lies in sub-block j = i / 32 and
 *   w_i = d * sc_j * q_i - dmin * m_j.
 * d*sc_j (17 bits), (d*sc_j)*q_i (22 bits) and dmin*m_j (17 bits) are exact in
 * f32; only the final subtraction rounds (to nearest even).
 * Pinned by: per-slot round trips (every sc/m slot x all 64 values, every
 * position x all 32 quants), second decoder, hand-worked blocks, closed
 * forms. */
void orc_dequant_block_q5_k(const uint8_t *blk, float *w)
{
    float d = half_at(blk + 0);
    float dmin = half_at(blk + 2);
    const uint8_t *scales = blk + 4;
    const uint8_t *qh = blk + 16;
    const uint8_t *qs = blk + 48;

    int sc[8], m[8];
    for (int j = 0; j < 8; ++j) {
        if (j < 4) {
            sc[j] = scales[j] & 63;
            m[j] = scales[j + 4] & 63;
        } else {
            sc[j] = (scales[j + 4] & 15) | ((scales[j - 4] >> 6) << 4);
            m[j] = (scales[j + 4] >> 4) | ((scales[j] >> 6) << 4);
        }
    }

    int q[256];
    for (int c = 0; c < 4; ++c) {
        for (int l = 0; l < 32; ++l) {
            uint8_t b = qs[32 * c + l];
            int b5lo = (qh[l] >> (2 * c)) & 1;
            int b5hi = (qh[l] >> (2 * c + 1)) & 1;
            q[64 * c + l] = (b & 15) + 16 * b5lo;
            q[64 * c + 32 + l] = (b >> 4) + 16 * b5hi;
        }
    }

    for (int i = 0; i < 256; ++i) {
        int j = i / 32;
        float t1 = d * (float)sc[j];
        float t2 = dmin * (float)m[j];
        w[i] = t1 * (float)q[i] - t2;
    }
}

/* ----------------------------------------------------------- matrices -- */

static int shape_ok(int fmt, int64_t rows, int64_t cols)
{
    int bw = orc_block_weights(fmt);
    if (bw == 0 || rows < 1 || cols < 1 || cols % bw != 0) return 0;
    return 1;
}

/* Dequantize row r of a dense row-major block matrix into out[cols]. */
static void dequant_row(int fmt, const uint8_t *W, int64_t cols, int64_t r, float *out)
{
    int bw = orc_block_weights(fmt);
    int bb = orc_block_bytes(fmt);
    int64_t nb = cols / bw;
    const uint8_t *row = W + r * nb * bb;
    for (int64_t b = 0; b < nb; ++b) {
        const uint8_t *blk = row + b * bb;
        float *o = out + b * bw;
        if (fmt == ORC_Q8_0) orc_dequant_block_q8_0(blk, o);
        else if (fmt == ORC_Q4_K) orc_dequant_block_q4_k(blk, o);
        else if (fmt == ORC_Q6_K) orc_dequant_block_q6_k(blk, o);
        else if (fmt == ORC_Q4_0) orc_dequant_block_q4_0(blk, o);
        else orc_dequant_block_q5_k(blk, o);
    }
}

int orc_dequant(int fmt, const uint8_t *W, int64_t rows, int64_t cols, float *out)
{
    if (!W || !out || !shape_ok(fmt, rows, cols)) return -1;
    for (int64_t r = 0; r < rows; ++r) dequant_row(fmt, W, cols, r, out + r * cols);
    return 0;
}

/* One output row for every token: f64 sum in index order, and the sum of
 * absolute products (the scale of the rounding error allowed to a kernel). */
static void row_dot(const float *w, int64_t cols, const float *x, int n_tok,
                    int64_t ystride, double *y, double *bound)
{
    for (int t = 0; t < n_tok; ++t) {
        const float *xt = x + (int64_t)t * cols;
        double acc = 0.0, mag = 0.0;
        for (int64_t i = 0; i < cols; ++i) {
            double p = (double)w[i] * (double)xt[i];
            acc += p;
            mag += fabs(p);
        }
        if (y) y[t * ystride] = acc;
        if (bound) bound[t * ystride] = mag;
    }
}

int orc_qmv(int fmt, const uint8_t *W, int64_t rows, int64_t cols,
            const float *x, int n_tok, double *y, double *bound, int nthreads)
{
    if (!W || !x || n_tok < 1 || !shape_ok(fmt, rows, cols)) return -1;
    if (nthreads < 1) nthreads = 1;
    int failed = 0;
#ifdef _OPENMP
#pragma omp parallel num_threads(nthreads)
#endif
    {
        float *wrow = (float *)malloc((size_t)cols * sizeof(float));
        if (!wrow) {
            failed = 1;
        } else {
#ifdef _OPENMP
#pragma omp for schedule(static)
#endif
            for (int64_t r = 0; r < rows; ++r) {
                dequant_row(fmt, W, cols, r, wrow);
                row_dot(wrow, cols, x, n_tok, rows, y ? y + r : NULL, bound ? bound + r : NULL);
            }
            free(wrow);
        }
    }
    return failed ? -1 : 0;
}

int orc_qmv_rows(int fmt, const uint8_t *W, int64_t rows, int64_t cols,
                 const int64_t *row_idx, int64_t n_rows,
                 const float *x, int n_tok, double *y, double *bound)
{
    if (!W || !x || !row_idx || n_tok < 1 || n_rows < 0 || !shape_ok(fmt, rows, cols)) return -1;
    float *wrow = (float *)malloc((size_t)cols * sizeof(float));
    if (!wrow) return -1;
    int rc = 0;
    for (int64_t k = 0; k < n_rows; ++k) {
        int64_t r = row_idx[k];
        if (r < 0 || r >= rows) { rc = -1; break; }
        dequant_row(fmt, W, cols, r, wrow);
        row_dot(wrow, cols, x, n_tok, n_rows, y ? y + k : NULL, bound ? bound + k : NULL);
    }
    free(wrow);
    return rc;
}

/* ----------------------------------------------------------------- MoE -- */

/* [BebeLM] §核心算子, MoE前馈网络: the router's activation is a sigmoid (not a
 * softmax), k = 4 experts of 32 are chosen, the per-expert bias takes part in
 * the choice only, and the chosen weights are normalised (norm_topk_prob).
 * The biased score is read as sigmoid(logit) + bias.
 * Pinned by: brute force over all C(32,4) subsets, bias = 0 reducing to the
 * top-4 logits, sum(g) = 1, hand-worked cases. */
int orc_route(const float *logits, const float *bias, int n_expert, int top_k,
              int32_t *ids, double *g, float *biased_out)
{
    if (!logits || !bias || !ids || !g || n_expert < 1 || top_k < 1 || top_k > n_expert)
        return -1;
    float *b = (float *)malloc((size_t)n_expert * sizeof(float));
    char *taken = (char *)calloc((size_t)n_expert, 1);
    if (!b || !taken) { free(b); free(taken); return -1; }

    for (int e = 0; e < n_expert; ++e) {
        float s = 1.0f / (1.0f + expf(-logits[e]));
        b[e] = s + bias[e];
        if (biased_out) biased_out[e] = b[e];
    }
    for (int k = 0; k < top_k; ++k) {
        int best = -1;
        for (int e = 0; e < n_expert; ++e) {
            if (taken[e]) continue;
            if (best < 0 || b[e] > b[best]) best = e; /* ties keep the lower index */
        }
        taken[best] = 1;
        ids[k] = best;
    }
    double total = 0.0;
    for (int k = 0; k < top_k; ++k) total += 1.0 / (1.0 + exp(-(double)logits[ids[k]]));
    for (int k = 0; k < top_k; ++k) g[k] = (1.0 / (1.0 + exp(-(double)logits[ids[k]]))) / total;

    free(b);
    free(taken);
    return 0;
}

double orc_silu(double z)
{
    return z / (1.0 + exp(-z));
}

int orc_moe_ffn(int fmt_gu, const uint8_t *gate_base, const uint8_t *up_base,
                int64_t gu_stride, int fmt_down, const uint8_t *down_base,
                int64_t down_stride, int n_expert, const int32_t *ids,
                const double *g, int n_sel, int64_t hidden, int64_t inter,
                const float *x, double *u, double *v, double *h, double *y)
{
    if (!gate_base || !up_base || !down_base || !ids || !g || !x || n_sel < 1)
        return -1;
    if (!shape_ok(fmt_gu, inter, hidden) || !shape_ok(fmt_down, hidden, inter)) return -1;
    for (int k = 0; k < n_sel; ++k)
        if (ids[k] < 0 || ids[k] >= n_expert) return -1;

    double *hk = (double *)malloc((size_t)n_sel * inter * sizeof(double));
    float *wrow = (float *)malloc((size_t)(hidden > inter ? hidden : inter) * sizeof(float));
    if (!hk || !wrow) { free(hk); free(wrow); return -1; }

    /* u_k = G x, v_k = U x, h_k = silu(u_k) * v_k */
    for (int k = 0; k < n_sel; ++k) {
        const uint8_t *G = gate_base + (int64_t)ids[k] * gu_stride;
        const uint8_t *U = up_base + (int64_t)ids[k] * gu_stride;
        for (int64_t r = 0; r < inter; ++r) {
            double uk = 0.0, vk = 0.0;
            dequant_row(fmt_gu, G, hidden, r, wrow);
            for (int64_t i = 0; i < hidden; ++i) uk += (double)wrow[i] * (double)x[i];
            dequant_row(fmt_gu, U, hidden, r, wrow);
            for (int64_t i = 0; i < hidden; ++i) vk += (double)wrow[i] * (double)x[i];
            double hv = orc_silu(uk) * vk;
            hk[k * inter + r] = hv;
            if (u) u[k * inter + r] = uk;
            if (v) v[k * inter + r] = vk;
            if (h) h[k * inter + r] = hv;
        }
    }
    /* y = sum_k g_k * D_k h_k */
    if (y) {
        for (int64_t r = 0; r < hidden; ++r) y[r] = 0.0;
        for (int k = 0; k < n_sel; ++k) {
            const uint8_t *D = down_base + (int64_t)ids[k] * down_stride;
            for (int64_t r = 0; r < hidden; ++r) {
                double acc = 0.0;
                dequant_row(fmt_down, D, inter, r, wrow);
                for (int64_t i = 0; i < inter; ++i) acc += (double)wrow[i] * hk[k * inter + i];
                y[r] += g[k] * acc;
            }
        }
    }
    free(hk);
    free(wrow);
    return 0;
}
