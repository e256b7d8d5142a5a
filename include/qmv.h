/*
 * qmv.h -- C ABI of libqmv.so: the decode-step matrix-vector product of a
 * GGUF block-quantized weight matrix (Q8_0, Q4_0, Q4_K, Q5_K, Q6_K) with f32
 * activations, dequantized on the fly, on one NVIDIA B200 (sm_100a).
 *
 * Sources (page title, section):
 *   BebeLM：纯Rust实现的端侧大模型推理引擎
 *     §量化格式支持 -- Q4_K: 256 weights per superblock in 144 bytes; Q6_K for
 *       sensitive tensors; dequantization happens at run time and activations
 *       stay f32.
 *     §核心算子 (MoE前馈网络) -- sigmoid router, top-k = 4 of 32 experts, the
 *       expert bias takes part in the selection only, weights normalised.
 *     §性能表现 -- decode is bound by memory bandwidth.
 *   FlareLLM：纯Rust打造的浏览器端LLM推理引擎
 *     §推理层面的深度优化 -- fused QKV and gate/up matvecs (43% fewer matvec
 *       calls per layer); n-gram speculative decoding (several tokens checked
 *       in one pass over the weights); zero-allocation forward pass.
 *     §计算路径的智能选择, §量化技术的全面支持 -- Q8_0, Q4_0 and the K-quants.
 *     §生态对比与定位 -- standard GGUF files.
 *
 * Block layouts (GGUF, little-endian, fp16 = IEEE binary16):
 *   Q8_0  32 weights / 34 B : d | q[32] int8                 w = d*q
 *   Q4_K 256 weights / 144 B: d | dmin | scales[12] | qs[128]
 *                             w = d*sc_j*q - dmin*m_j, j = sub-block of 32
 *   Q6_K 256 weights / 210 B: ql[128] | qh[64] | scales[16] int8 | d
 *                             w = d*scales[i/16]*(q - 32), q = 6 bits
 *   Q4_0  32 weights / 18 B : d | qs[16]; byte j holds weight j (low nibble)
 *                             and weight j+16 (high nibble);  w = d*(q - 8)
 *   Q5_K 256 weights / 176 B: d | dmin | scales[12] (as Q4_K) | qh[32] | qs[128]
 *                             (as Q4_K); the fifth bit of weight 64c + l is
 *                             bit 2c of qh[l], of weight 64c + 32 + l bit 2c+1;
 *                             w = d*sc_j*q - dmin*m_j
 * A matrix is rows x cols weights stored densely row-major: row r starts at
 * byte r * (cols / block_weights) * block_bytes; no padding.
 *
 * Conventions shared by every entry point:
 *   - Every array pointer is a DEVICE pointer owned by the caller (for
 *     example torch.empty(..., device="cuda").data_ptr()); the library keeps
 *     no reference after the call returns.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Work is
 *     enqueued asynchronously on it; outputs are complete in stream order.
 *   - The library allocates no memory during any call; intermediates (the
 *     SwiGLU activations of moe_ffn) live in caller-provided buffers.
 *   - Outputs are fully overwritten, never accumulated into.
 *   - Argument errors are detected on the host and returned before anything
 *     is enqueued; outputs are then left untouched.  No call aborts.
 *   - Alignment: W (every expert base and expert stride) 16 B, x 16 B,
 *     y / out 4 B.
 *   - The arithmetic is f32: dequantized weights are exact f32 values, dot
 *     products accumulate in f32 (order unspecified, deterministic for a
 *     given shape).  There is no CPU fallback and no other backend.
 *   - Thread safety: calls may be made from several host threads.  Global
 *     state: a per-device properties cache, the programmatic-dependent-launch
 *     switch (qmv_set_pdl), and per device the sticky error word read by
 *     qmv_check(), qmv_argmax's workspace and the scratch array of
 *     moe_ffn_static.
 */
#ifndef QMV_H
#define QMV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t, without including the CUDA headers. */
typedef struct CUstream_st *qmv_stream_t;

typedef enum { QMV_Q8_0 = 0, QMV_Q4_K = 1, QMV_Q6_K = 2, QMV_Q4_0 = 3, QMV_Q5_K = 4 } qmv_fmt;

typedef enum {
    QMV_OK = 0,
    QMV_ERR_NULL = -1,    /* a required pointer is NULL                         */
    QMV_ERR_FMT = -2,     /* fmt is not one of qmv_fmt                           */
    QMV_ERR_SHAPE = -3,   /* rows < 1, cols < 1, cols % block_weights != 0, or a
                             size above the limits below                        */
    QMV_ERR_ALIGN = -4,   /* a pointer or stride breaks the alignment rules      */
    QMV_ERR_NTOK = -5,    /* n_tok outside [1, QMV_MAX_NTOK]                     */
    QMV_ERR_NSEL = -6,    /* n_sel / top_k outside [1, min(n_expert, 8)], or
                             n_expert outside [1, QMV_MAX_EXPERTS]              */
    QMV_ERR_CUDA = -7,    /* a CUDA call or a kernel launch failed               */
    QMV_ERR_DEVICE = -8,  /* no usable CUDA device, or a device-side error was
                             recorded (see qmv_check)                            */
} qmv_status;

#define QMV_MAX_NTOK 8
#define QMV_MAX_SEL 8
#define QMV_MAX_EXPERTS 1024
#define QMV_MAX_ROWS 2147483647LL   /* rows of one matrix                       */
#define QMV_MAX_COLS 1048576LL      /* weights per row                          */

/* Device error bits reported by qmv_check(). */
#define QMV_DEVERR_EXPERT_ID 1      /* an expert id was outside [0, n_expert); that
                                       expert's contribution was dropped        */
#define QMV_DEVERR_TIMEOUT 2        /* a pipeline wait gave up (bounded wait)   */
#define QMV_DEVERR_DRAIN 4          /* after a timeout, a CTA also gave up waiting for
                                       its own copies in flight and exited: they may
                                       still land in shared memory reused by later
                                       kernels, so later results on this device are
                                       suspect (recreate the context to be sure)   */

/* y[rows] = W x.  x: f32 [cols]; y: f32 [rows].
 * One launch covers a whole fused projection: pass the row-concatenation of
 * Q, K and V (or of gate and up) as W (FlareLLM page, §推理层面的深度优化).
 * Returns QMV_OK or a qmv_status error. */
int qmv_f32(int fmt, const void *W_blocks, int64_t rows, int64_t cols,
            const float *x, float *y, qmv_stream_t stream);

/* One matvec of a grouped launch (see qmv_multi). */
typedef struct {
    const void *W_blocks;   /* device, 16-byte aligned, rows x cols weights    */
    int64_t rows;
    int64_t cols;
    const float *x;         /* device f32 [n_tok][cols], 16-byte aligned       */
    float *y;               /* device f32 [n_tok][rows], 4-byte aligned        */
} qmv_task;

#define QMV_MAX_TASKS 4096

/* Several independent matvecs of one format and token count in as few
 * launches as possible: y_t = W_t x_t for every task t (same layouts as
 * qmv_batched).  The tasks run concurrently and in no defined order, so no
 * task may write memory another task of the call reads; the call as a whole
 * is ordered in `stream` like any other.  Each task's rows are split into
 * CTAs of roughly equal byte counts sized to the whole batch, so the CTAs of
 * all tasks stream together and the launch-to-launch latency of a chain of
 * small matvecs disappears.  `tasks` is a host array of n_tasks entries
 * (1 <= n_tasks <= QMV_MAX_TASKS), read during the call only. */
int qmv_multi(int fmt, int n_tok, const qmv_task *tasks, int n_tasks, qmv_stream_t stream);

/* One-token matvecs of one format executed IN ORDER, the way a decode step
 * runs its projections layer after layer (BebeLM：纯Rust实现的端侧大模型推理引擎,
 * §核心算子 and §性能表现: every layer's matvecs each decode step): task t+1
 * starts only after every row of task t is written, so a task's x may be the
 * y of any earlier task of the same call (tasks' n_tok is 1: x f32 [cols],
 * y f32 [rows]).  Each task is one streaming-kernel launch, ordered by
 * programmatic dependent launch (a kernel reads its x only after the previous
 * one has finished), and each launch, once its own weight copies are issued,
 * starts moving the next task's weights into L2, so the next launch reads them
 * from there while HBM already streams the one after.  The call keeps no
 * state between calls: calls on different streams may overlap.  A task shape
 * that the streaming kernel does not take turns the whole call into one
 * qmv_f32 call per task, in order.  `tasks` is a host array of
 * n_tasks entries (1 <= n_tasks <= QMV_MAX_TASKS), read during the call only.
 * Errors as qmv_multi. */
int qmv_chain(int fmt, const qmv_task *tasks, int n_tasks, qmv_stream_t stream);

/* Multi-token variant for speculative verification (FlareLLM page,
 * §推理层面的深度优化: n-gram speculative decoding): every weight is read once
 * and applied to n_tok activation vectors.
 * x: f32 [n_tok][cols] (token-major); y: f32 [n_tok][rows]; 1 <= n_tok <= 8. */
int qmv_batched(int fmt, const void *W_blocks, int64_t rows, int64_t cols,
                const float *x, float *y, int n_tok, qmv_stream_t stream);

/* MoE router on the device, no host round trip (BebeLM page, §核心算子):
 *   s_e = sigmoid(logits[e]),  b_e = s_e + bias[e]   (f32)
 *   ids_out[k] = the top_k experts by b, in descending b (ties to the lower
 *                index);  g_out[k] = s_{ids[k]} / sum_j s_{ids[j]}.
 * logits, bias: f32 [n_expert]; ids_out: int32 [top_k]; g_out: f32 [top_k].
 * 1 <= top_k <= min(n_expert, 8), n_expert <= QMV_MAX_EXPERTS. */
int moe_route(const float *logits, const float *bias, int n_expert, int top_k,
              int32_t *ids_out, float *g_out, qmv_stream_t stream);

/* Expert-indexed grouped matvec.  Expert e's matrix (rows x cols, format fmt)
 * starts at expert_blocks + e * expert_stride_bytes; the n_sel expert ids are
 * read on the device from expert_ids (int32 [n_sel]), so the call can follow
 * moe_route without a host synchronisation.
 * x_k = x + k * x_stride (x_stride in floats; 0 = one shared x [cols]).
 *   gate_w == NULL: y[k][r] = (W_{ids[k]} x_k)[r]           y: f32 [n_sel][rows]
 *   gate_w != NULL: y[r] = sum_k gate_w[k] * (W_{ids[k]} x_k)[r]  y: f32 [rows]
 *                   (gate_w: device f32 [n_sel]; summed in k order)
 * An id outside [0, n_expert) contributes zero and sets QMV_DEVERR_EXPERT_ID.
 * 1 <= n_sel <= min(n_expert, 8).  expert_stride_bytes must be a multiple of
 * 16 and at least the matrix size. */
int moe_qmv(int fmt, const void *expert_blocks, int64_t expert_stride_bytes, int n_expert,
            const int32_t *expert_ids, int n_sel, int64_t rows, int64_t cols,
            const float *x, int64_t x_stride, const float *gate_w, float *y,
            qmv_stream_t stream);

/* One MoE SwiGLU FFN step for the n_sel routed experts (BebeLM page, §核心算子):
 *   h_k = silu(G_{ids[k]} x) * (U_{ids[k]} x)        -> h_scratch f32 [n_sel][inter]
 *   y   = sum_k g[k] * D_{ids[k]} h_k                 -> y f32 [hidden]
 * G and U of expert e: [inter x hidden] in fmt_gu at gate_blocks / up_blocks
 * + e * gu_stride_bytes; D of expert e: [hidden x inter] in fmt_down at
 * down_blocks + e * down_stride_bytes.  x: f32 [hidden]; g: f32 [n_sel]
 * (e.g. from moe_route).  silu(z) = z / (1 + exp(-z)).  Two launches, no host
 * synchronisation; h_scratch is caller-owned scratch and is overwritten. */
int moe_ffn(int fmt_gu, const void *gate_blocks, const void *up_blocks,
            int64_t gu_stride_bytes, int fmt_down, const void *down_blocks,
            int64_t down_stride_bytes, int n_expert, const int32_t *expert_ids,
            const float *g, int n_sel, int64_t hidden, int64_t inter,
            const float *x, float *h_scratch, float *y, qmv_stream_t stream);

/* The MoE FFN step with its router, in one launch where the shapes allow
 * (BebeLM page, §核心算子, MoE前馈网络): moe_route on (logits, bias, n_expert,
 * top_k) -- ids_out, g_out as moe_route writes them, the same values -- then
 * moe_ffn with those ids and weights (n_sel = top_k): h_scratch
 * f32 [top_k][inter] holds the SwiGLU activations, y f32 [hidden] the result.
 * When both matrices have one format, expert rows are at most 2048 columns,
 * n_expert <= 256 and the rows are 16-byte multiples in pairs, one
 * cooperative launch does it all: every CTA routes on its own, streams the
 * routed gate/up rows and then the routed down rows through one pipeline, and
 * the CTAs meet once, at a grid barrier, between the two products (h complete).
 * Otherwise moe_route and moe_ffn run in turn.  `workspace`:
 * QMV_MOE_WS_BYTES of caller-owned device memory (8-byte aligned) that must be
 * zero before the first call and that every completed call leaves zero again
 * (the barrier's counters); calls that may overlap on the GPU need workspaces
 * of their own.  Errors as moe_route and moe_ffn. */
#define QMV_MOE_WS_BYTES 16
int moe_ffn_routed(const float *logits, const float *bias, int n_expert, int top_k,
                   int fmt_gu, const void *gate_blocks, const void *up_blocks,
                   int64_t gu_stride_bytes, int fmt_down, const void *down_blocks,
                   int64_t down_stride_bytes, int64_t hidden, int64_t inter, const float *x,
                   int32_t *ids_out, float *g_out, float *h_scratch, float *y, void *workspace,
                   qmv_stream_t stream);

/* moe_ffn without a caller-provided scratch buffer, for callers that cannot
 * allocate device memory: code running while a stream is being captured into
 * a CUDA graph (where cudaMalloc is not allowed), plugins and callbacks that
 * are handed only their input and output buffers, and real-time paths that
 * must not take an allocator's latency or locks.  (The pages have no
 * counterpart; this is a usage variant of the same MoE step.)
 * The SwiGLU activations go to a file-scope device array of
 * QMV_STATIC_H_FLOATS floats (512 KiB) that every GPU which loads the library
 * holds until the process exits; n_sel * inter above that is rejected with
 * QMV_ERR_SHAPE.  Nothing is allocated by the call.  The first call on a
 * device looks up the array's device address (a host call, no allocation):
 * make that first call before capturing a stream.  All calls share the one
 * array, which keeps the last call's contents (every call overwrites the part
 * it uses before reading it), so calls that can overlap on the GPU -- on two
 * streams of one device, say -- race and must be serialised by the caller.
 * Arguments and results are those of moe_ffn. */
#define QMV_STATIC_H_FLOATS (8 * 16384)
int moe_ffn_static(int fmt_gu, const void *gate_blocks, const void *up_blocks,
                   int64_t gu_stride_bytes, int fmt_down, const void *down_blocks,
                   int64_t down_stride_bytes, int n_expert, const int32_t *expert_ids,
                   const float *g, int n_sel, int64_t hidden, int64_t inter,
                   const float *x, float *y, qmv_stream_t stream);

/* Greedy next-token choice on the device (FlareLLM page, §推理层面的深度优化:
 * greedy decoding of the vocabulary projection): y = W x as qmv_batched (the
 * logits are kept in the caller's y, f32 [n_tok][rows]), and
 * idx_out[t] = the row of the largest y[t][row] -- IEEE > on f32, ties to
 * the lower row, NaN values skipped, -1 if every value of the token is NaN.
 * idx_out: device int32 [n_tok], 4-byte aligned.  rows <= INT32_MAX.
 * With one token on the shapes the one-token streaming kernel takes (rows of
 * at most 2048 columns) the choice is fused into the projection: every CTA
 * folds the best of its rows into a 64-bit key while it writes them, and the
 * last CTA writes idx -- one launch.  Otherwise a second launch scans y.
 * Either way the choice is deterministic (an order-independent atomic max
 * over keys: the value's order-preserving bits high, the complemented row
 * low).
 * The keys and arrival counters live in `workspace`, QMV_ARGMAX_WS_BYTES of
 * caller-owned device memory (8-byte aligned) that must be zero before the
 * first call and that every completed call leaves zero again; calls that may
 * overlap on the GPU need workspaces of their own.  Errors as qmv_batched,
 * QMV_ERR_NULL for a NULL workspace. */
#define QMV_ARGMAX_WS_BYTES 128
int qmv_argmax_ws(int fmt, const void *W_blocks, int64_t rows, int64_t cols,
                  const float *x, float *y, int n_tok, int32_t *idx_out, void *workspace,
                  qmv_stream_t stream);

/* qmv_argmax_ws with the library's own workspace on the current device: do
 * not run two qmv_argmax calls on one device at the same time (use
 * qmv_argmax_ws with separate workspaces for that). */
int qmv_argmax(int fmt, const void *W_blocks, int64_t rows, int64_t cols,
               const float *x, float *y, int n_tok, int32_t *idx_out, qmv_stream_t stream);

/* Dequantize the whole matrix to f32: out[rows][cols].  The values are
 * bit-exact f32 evaluations of the block formulas above (every product in
 * them is exact in f32; Q4_K and Q5_K round once, in the subtraction). */
int qmv_dequant(int fmt, const void *W_blocks, int64_t rows, int64_t cols,
                float *out, qmv_stream_t stream);

/* Synchronises `stream`, then reads and clears the sticky device error word
 * of the current device.  Returns QMV_OK, QMV_ERR_CUDA if the synchronisation
 * failed, or QMV_ERR_DEVICE if an error bit was set (the bits are stored in
 * *dev_err_out when it is not NULL). */
int qmv_check(qmv_stream_t stream, int *dev_err_out);

/* Static, never-NULL description of a qmv_status value. */
const char *qmv_strerror(int status);

/* Description of the CUDA error behind the last QMV_ERR_CUDA returned on the
 * calling host thread ("no error" if there was none). */
const char *qmv_last_cuda_error(void);

/* Bytes and weights per block of a format; 0 for an unknown format. */
size_t qmv_block_bytes(int fmt);
int qmv_block_weights(int fmt);

/* Programmatic dependent launch for the matvec launches (process-wide, off by
 * default).  When enabled, a matvec launch may start -- and begin streaming
 * its weight blocks into shared memory -- while the previous kernel in the
 * stream is still running; it waits for that kernel to finish before it reads
 * x, expert ids or gate weights and before it writes any output.  This hides
 * the launch gap between back-to-back matvecs of a decode step.  Enable it
 * only when no kernel still in flight on the stream writes the weight blocks
 * (true for inference weights loaded once).  qmv_get_pdl returns the setting. */
void qmv_set_pdl(int enable);
int qmv_get_pdl(void);

/* Test hook: which kernel served the calling host thread's most recent
 * matvec call (qmv_f32, qmv_batched, qmv_multi, qmv_chain, moe_qmv, moe_ffn,
 * qmv_argmax), so tests can show that each kernel path is exercised.
 * QMV_KERNEL_NONE before the first such call on the thread. */
#define QMV_KERNEL_NONE 0
#define QMV_KERNEL_WARP_RING 1      /* one to four tokens, per-warp copy rings   */
#define QMV_KERNEL_GENERAL 2        /* general pipeline (groups, grouped launches) */
#define QMV_KERNEL_TENSOR_CORE 3    /* three to eight tokens, mma.sync          */
#define QMV_KERNEL_STREAM 4         /* one token, producer warp + whole-row stages */
int qmv_debug_last_kernel(void);

/* Test hook for host-side failure handling: the next `count` launches made by
 * this library fail with QMV_ERR_CUDA without reaching the GPU. */
void qmv_debug_fail_next_launches(int count);

/* Test hook for the device-side failure path: while bytes > 0, the
 * streaming, warp-ring and tensor-core launches (qmv_f32 / qmv_batched on the
 * shapes that take them, qmv_chain) expect `bytes` more per copied tile than
 * they copy, so every stage wait runs into its bound (about a second), records
 * QMV_DEVERR_TIMEOUT (and, where a kernel then also gives up waiting for its
 * own copies, QMV_DEVERR_DRAIN) for qmv_check, and the kernel still finishes;
 * results are then undefined.  0 (the default) turns it off.  Not for
 * production. */
void qmv_debug_short_copies(int bytes);

#ifdef __cplusplus
}
#endif
#endif /* QMV_H */
