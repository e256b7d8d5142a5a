// qmv_device.cuh -- device building blocks of the sm_100a quantized matvec:
// shared-memory / mbarrier / bulk-copy PTX wrappers, the per-format
// superblock decode units, and the multi-row warp reduction.
//
// Block layouts (GGUF, little-endian) -- BebeLM：纯Rust实现的端侧大模型推理引擎,
// §量化格式支持 (Q4_K: 256 weights in 144 bytes; Q6_K for sensitive tensors;
// run-time dequantization with f32 activations) and FlareLLM：纯Rust打造的浏览器端
// LLM推理引擎, §计算路径的智能选择 (Q8_0):
//   Q8_0  34 B : d(fp16) | q[32] int8                       w = d*q
//   Q4_K 144 B : d | dmin | scales[12] | qs[128]            w = d*sc_j*q - dmin*m_j
//   Q6_K 210 B : ql[128] | qh[64] | scales[16] int8 | d      w = d*scales[i/16]*(q-32)
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace qmv {

enum { FMT_Q8_0 = 0, FMT_Q4_K = 1, FMT_Q6_K = 2 };

template <int FMT> struct Fmt;
template <> struct Fmt<FMT_Q8_0> { static constexpr int BW = 32;  static constexpr int BB = 34; };
template <> struct Fmt<FMT_Q4_K> { static constexpr int BW = 256; static constexpr int BB = 144; };
template <> struct Fmt<FMT_Q6_K> { static constexpr int BW = 256; static constexpr int BB = 210; };

// ------------------------------------------------------------ PTX wrappers --

__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t lds_u32(uint32_t a)
{
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}

__device__ __forceinline__ uint32_t lds_u16(uint32_t a)
{
    unsigned short v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
    return v;
}

__device__ __forceinline__ uint4 lds_v4(uint32_t a)
{
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}

__device__ __forceinline__ void sts_u16(uint32_t a, uint32_t v)
{
    asm volatile("st.shared.u16 [%0], %1;" :: "r"(a), "h"((unsigned short)v) : "memory");
}

__device__ __forceinline__ void sts_f32(uint32_t a, float v)
{
    asm volatile("st.shared.f32 [%0], %1;" :: "r"(a), "f"(v) : "memory");
}

__device__ __forceinline__ float lds_f32(uint32_t a)
{
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a) : "memory");
    return v;
}

// 4*N bytes starting at a 2-byte-aligned shared address, as N little-endian
// words.  Reads up to 4 bytes past the last requested byte (stages are padded).
template <int N>
__device__ __forceinline__ void lds_words_a2(uint32_t a, uint32_t (&w)[N])
{
    const uint32_t base = a & ~3u;
    const uint32_t sh = (a & 2u) * 8u;   // 0 or 16
    uint32_t prev = lds_u32(base);
#pragma unroll
    for (int i = 0; i < N; ++i) {
        const uint32_t nx = lds_u32(base + 4u * (i + 1));
        w[i] = __funnelshift_r(prev, nx, sh);
        prev = nx;
    }
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("{\n\t.reg .b64 st;\n\t"
                 "mbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" :: "r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t tx)
{
    asm volatile("{\n\t.reg .b64 st;\n\t"
                 "mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}"
                 :: "r"(bar), "r"(tx) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Waits for the phase with the given parity to complete; gives up after about
// one second of wall time and returns false (the caller records the error).
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 0u && global_timer_ns() - t0 > 1000000000ull) return false;
    }
}

// L2 eviction policy for streamed-once weight bytes.
__device__ __forceinline__ uint64_t policy_evict_first()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// One 1-D bulk copy global -> this CTA's shared memory, completing on `bar`.
// dst, src 16-byte aligned, bytes a multiple of 16.  Local memory only.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes,
                                        uint32_t bar, uint64_t pol)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
                 " [%0], [%1], %2, [%3], %4;"
                 :: "r"(dst), "l"(src), "r"(bytes), "r"(bar), "l"(pol) : "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads)
{
    asm volatile("bar.sync %0, %1;" :: "r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ float half_bits_to_float(uint32_t bits)
{
    return __half2float(__ushort_as_half(static_cast<unsigned short>(bits & 0xFFFFu)));
}

// ------------------------------------------------- multi-row warp reduction --
// v[V] (V a power of two <= 32) holds this lane's partial sums of V different
// outputs.  Each butterfly step halves the number of values a lane carries by
// exchanging the half it does not keep; after log2(V) steps a lane carries one
// value and the remaining steps finish the sum.  Costs V - 1 + 5 - log2(V)
// shuffles instead of 5 V.  On return, lane L holds in v[0] the full sum of
// output index (L >> (5 - log2 V)).
template <int V>
__device__ __forceinline__ void warp_transpose_reduce(float (&v)[V], int lane)
{
    static_assert(V >= 1 && V <= 32 && (V & (V - 1)) == 0, "V must be a power of two <= 32");
#pragma unroll
    for (int step = 0; (1 << step) < V; ++step) {
        const int o = 16 >> step;
        const int half = V >> (step + 1);
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int k = 0; k < half; ++k) {
            const float send = upper ? v[k] : v[k + half];
            const float keep = upper ? v[k + half] : v[k];
            v[k] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, o);
        }
    }
    constexpr int LOG = (V >= 32) ? 5 : (V >= 16) ? 4 : (V >= 8) ? 3 : (V >= 4) ? 2 : (V >= 2) ? 1 : 0;
#pragma unroll
    for (int o = 16 >> LOG; o >= 1; o >>= 1) v[0] += __shfl_xor_sync(0xFFFFFFFFu, v[0], o);
}

// ---------------------------------------------------------- decode units --
// A "slice" is 32 weights of one row handled by one lane.  Each unit below
// reads its slice's bytes from shared memory, and for every token t adds the
// slice's contribution sum_i w_i * x[t][col_i] to acc[t].  The x values come
// from an accessor xf(t, q) returning the q-th group of 4 x values (q = 0..7)
// in the slice's own column order, documented per format.  The weights are
// never materialised: per scale group the unit forms sum q*x (and sum x for
// the Q4_K min term) and applies the scales once.

// Q8_0: slice = one block at shared address blk (2-byte aligned).
// Column order: the block's 32 weights in order.
template <int NTOK, class XF>
__device__ __forceinline__ void slice_q8_0(uint32_t blk, XF &&xf, float (&acc)[NTOK])
{
    const float d = half_bits_to_float(lds_u16(blk));
    uint32_t w[8];
    lds_words_a2<8>(blk + 2, w);
    float s[NTOK];
#pragma unroll
    for (int t = 0; t < NTOK; ++t) s[t] = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const float q0 = (float)(int)(int8_t)(w[q] & 0xFFu);
        const float q1 = (float)(int)(int8_t)((w[q] >> 8) & 0xFFu);
        const float q2 = (float)(int)(int8_t)((w[q] >> 16) & 0xFFu);
        const float q3 = (float)(int)(int8_t)(w[q] >> 24);
#pragma unroll
        for (int t = 0; t < NTOK; ++t) {
            const float4 x = xf(t, q);
            s[t] = fmaf(q0, x.x, s[t]);
            s[t] = fmaf(q1, x.y, s[t]);
            s[t] = fmaf(q2, x.z, s[t]);
            s[t] = fmaf(q3, x.w, s[t]);
        }
    }
#pragma unroll
    for (int t = 0; t < NTOK; ++t) acc[t] = fmaf(d, s[t], acc[t]);
}

// Q4_K sub-block scale / min j (0..7) from the 12 scale bytes held in three
// words (bytes 0-3, 4-7, 8-11):
//   j < 4 : sc = b[j] & 63,                        m = b[j+4] & 63
//   j >= 4: sc = (b[j+4] & 15) | ((b[j-4] >> 6) << 4),
//           m  = (b[j+4] >> 4) | ((b[j] >> 6) << 4)
__device__ __forceinline__ uint32_t scale_byte(uint32_t s0, uint32_t s1, uint32_t s2, int idx)
{
    const uint32_t word = idx < 4 ? s0 : (idx < 8 ? s1 : s2);
    return (word >> ((idx & 3) * 8)) & 0xFFu;
}

__device__ __forceinline__ void q4k_scale_min(uint32_t s0, uint32_t s1, uint32_t s2, int j,
                                              uint32_t &sc, uint32_t &m)
{
    if (j < 4) {
        sc = scale_byte(s0, s1, s2, j) & 63u;
        m = scale_byte(s0, s1, s2, j + 4) & 63u;
    } else {
        const uint32_t b = scale_byte(s0, s1, s2, j + 4);
        sc = (b & 15u) | ((scale_byte(s0, s1, s2, j - 4) >> 6) << 4);
        m = (b >> 4) | ((scale_byte(s0, s1, s2, j) >> 6) << 4);
    }
}

// Q4_K: slice k (0..7) of the superblock at shared address sb (16-byte
// aligned).  Chunk c = k/2 and half hf = k%2 select qs bytes [32c+16hf, +16):
// their low nibbles are weights 64c+16hf+[0,16) (sub-block 2c), their high
// nibbles weights 64c+32+16hf+[0,16) (sub-block 2c+1).
// Column order: groups q = 0..3 are the 16 low-nibble columns, q = 4..7 the
// 16 high-nibble columns.  xsum(t, 0 / 1) returns the sum of the 16 x values
// of the low / high run (precomputed when x is held in registers).
template <int NTOK, class XF, class XS>
__device__ __forceinline__ void slice_q4_k(uint32_t sb, int k, XF &&xf, XS &&xsum, float (&acc)[NTOK])
{
    const uint4 hdr = lds_v4(sb);
    const uint4 qv = lds_v4(sb + 16u + 16u * (uint32_t)k);
    const float d = half_bits_to_float(hdr.x);
    const float dmin = half_bits_to_float(hdr.x >> 16);
    const int c = k >> 1;
    uint32_t sc0, m0, sc1, m1;
    q4k_scale_min(hdr.y, hdr.z, hdr.w, 2 * c, sc0, m0);
    q4k_scale_min(hdr.y, hdr.z, hdr.w, 2 * c + 1, sc1, m1);
    const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
    float slo[NTOK], shi[NTOK];
#pragma unroll
    for (int t = 0; t < NTOK; ++t) { slo[t] = 0.f; shi[t] = 0.f; }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint32_t wd = qw[q];
        float lo[4], hi[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            lo[e] = (float)((wd >> (8 * e)) & 15u);
            hi[e] = (float)((wd >> (8 * e + 4)) & 15u);
        }
#pragma unroll
        for (int t = 0; t < NTOK; ++t) {
            const float4 xl = xf(t, q);
            const float4 xh = xf(t, q + 4);
            slo[t] = fmaf(lo[0], xl.x, slo[t]);
            slo[t] = fmaf(lo[1], xl.y, slo[t]);
            slo[t] = fmaf(lo[2], xl.z, slo[t]);
            slo[t] = fmaf(lo[3], xl.w, slo[t]);
            shi[t] = fmaf(hi[0], xh.x, shi[t]);
            shi[t] = fmaf(hi[1], xh.y, shi[t]);
            shi[t] = fmaf(hi[2], xh.z, shi[t]);
            shi[t] = fmaf(hi[3], xh.w, shi[t]);
        }
    }
    const float dsc0 = d * (float)sc0, dsc1 = d * (float)sc1;
    const float dm0 = dmin * (float)m0, dm1 = dmin * (float)m1;
#pragma unroll
    for (int t = 0; t < NTOK; ++t) {
        float a = acc[t];
        a = fmaf(dsc0, slo[t], a);
        a = fmaf(dsc1, shi[t], a);
        a = fmaf(-dm0, xsum(t, 0), a);
        a = fmaf(-dm1, xsum(t, 1), a);
        acc[t] = a;
    }
}

// Q6_K: slice k (0..7) of the superblock at shared address sb (2-byte
// aligned).  Half h = k/4 and l0 = 8*(k%4): the slice holds weights
// 128h + 32t + l0 + e for t = 0..3, e = 0..7, whose low 4 bits are in
// ql[64h + l0 + e] (t = 0 low nibble, t = 2 high nibble) and
// ql[64h + 32 + l0 + e] (t = 1 low, t = 3 high), and whose high 2 bits are
// bits 2t..2t+1 of qh[32h + l0 + e]; their scale is scales[8h + 2t + l0/16].
// Column order: group q = 2t + (e / 4).
template <int NTOK, class XF>
__device__ __forceinline__ void slice_q6_k(uint32_t sb, int k, XF &&xf, float (&acc)[NTOK])
{
    const int h = k >> 2;
    const int l0 = 8 * (k & 3);
    uint32_t A[2], B[2], H[2];
    lds_words_a2<2>(sb + (uint32_t)(64 * h + l0), A);
    lds_words_a2<2>(sb + (uint32_t)(64 * h + 32 + l0), B);
    lds_words_a2<2>(sb + 128u + (uint32_t)(32 * h + l0), H);
    uint32_t S[4];
    lds_words_a2<4>(sb + 192u, S);                 // scales[0..15]
    const float d = half_bits_to_float(lds_u16(sb + 208u));
    float scl[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const int idx = 8 * h + 2 * t + (l0 >> 4);
        const int wi = idx >> 2;
        const uint32_t word = wi == 0 ? S[0] : wi == 1 ? S[1] : wi == 2 ? S[2] : S[3];
        scl[t] = (float)(int)(int8_t)((word >> ((idx & 3) * 8)) & 0xFFu);
    }
    float st[4][NTOK];
#pragma unroll
    for (int t = 0; t < 4; ++t)
#pragma unroll
        for (int n = 0; n < NTOK; ++n) st[t][n] = 0.f;
#pragma unroll
    for (int g = 0; g < 2; ++g) {
        float qf[4][4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const uint32_t a = (A[g] >> (8 * e)) & 0xFFu;
            const uint32_t b = (B[g] >> (8 * e)) & 0xFFu;
            const uint32_t hh = (H[g] >> (8 * e)) & 0xFFu;
            qf[0][e] = (float)((int)((a & 15u) | ((hh & 3u) << 4)) - 32);
            qf[1][e] = (float)((int)((b & 15u) | (((hh >> 2) & 3u) << 4)) - 32);
            qf[2][e] = (float)((int)((a >> 4) | (((hh >> 4) & 3u) << 4)) - 32);
            qf[3][e] = (float)((int)((b >> 4) | (((hh >> 6) & 3u) << 4)) - 32);
        }
#pragma unroll
        for (int t = 0; t < 4; ++t) {
#pragma unroll
            for (int n = 0; n < NTOK; ++n) {
                const float4 x = xf(n, 2 * t + g);
                float s = st[t][n];
                s = fmaf(qf[t][0], x.x, s);
                s = fmaf(qf[t][1], x.y, s);
                s = fmaf(qf[t][2], x.z, s);
                s = fmaf(qf[t][3], x.w, s);
                st[t][n] = s;
            }
        }
    }
#pragma unroll
    for (int n = 0; n < NTOK; ++n) {
        float s = 0.f;
#pragma unroll
        for (int t = 0; t < 4; ++t) s = fmaf(scl[t], st[t][n], s);
        acc[n] = fmaf(d, s, acc[n]);
    }
}

// Column (within the row) of group q of slice s, per format.
template <int FMT>
__device__ __forceinline__ int slice_group_col(int s, int q)
{
    if (FMT == FMT_Q8_0) {
        return 32 * s + 4 * q;
    } else if (FMT == FMT_Q4_K) {
        const int sb = s >> 3, k = s & 7, c = k >> 1, hf = k & 1;
        return 256 * sb + 64 * c + 16 * hf + (q < 4 ? 4 * q : 32 + 4 * (q - 4));
    } else {
        const int sb = s >> 3, k = s & 7, h = k >> 2, l0 = 8 * (k & 3);
        return 256 * sb + 128 * h + 32 * (q >> 1) + l0 + 4 * (q & 1);
    }
}

// ----------------------------------------------------- whole-block dequant --
// Exact f32 weights of one block (used by the dequant-only entry point).

__device__ __forceinline__ void dequant_block_q8_0(const uint8_t *blk, float *out)
{
    const float d = half_bits_to_float(blk[0] | (blk[1] << 8));
    for (int i = 0; i < 32; ++i) out[i] = d * (float)(int)(int8_t)blk[2 + i];
}

__device__ __forceinline__ void dequant_block_q4_k(const uint8_t *blk, float *out)
{
    const float d = half_bits_to_float(blk[0] | (blk[1] << 8));
    const float dmin = half_bits_to_float(blk[2] | (blk[3] << 8));
    uint32_t s[3];
    for (int w = 0; w < 3; ++w)
        s[w] = blk[4 + 4 * w] | (blk[5 + 4 * w] << 8) | (blk[6 + 4 * w] << 16) | ((uint32_t)blk[7 + 4 * w] << 24);
    for (int j = 0; j < 8; ++j) {
        uint32_t sc, m;
        q4k_scale_min(s[0], s[1], s[2], j, sc, m);
        const float dsc = d * (float)sc;    // exact
        const float dm = dmin * (float)m;   // exact
        const int c = j >> 1, hi = j & 1;
        for (int l = 0; l < 32; ++l) {
            const uint32_t b = blk[16 + 32 * c + l];
            const uint32_t q = hi ? (b >> 4) : (b & 15u);
            out[32 * j + l] = __fsub_rn(__fmul_rn(dsc, (float)q), dm);   // one rounding
        }
    }
}

__device__ __forceinline__ void dequant_block_q6_k(const uint8_t *blk, float *out)
{
    const float d = half_bits_to_float(blk[208] | (blk[209] << 8));
    for (int i = 0; i < 256; ++i) {
        const int h = i >> 7, t = (i >> 5) & 3, l = i & 31;
        const uint32_t lb = blk[64 * h + l + 32 * (t & 1)];
        const uint32_t low = (t < 2) ? (lb & 15u) : (lb >> 4);
        const uint32_t high = (blk[128 + 32 * h + l] >> (2 * t)) & 3u;
        const int q = (int)(low | (high << 4)) - 32;
        const float ds = d * (float)(int)(int8_t)blk[192 + (i >> 4)];
        out[i] = ds * (float)q;
    }
}

}  // namespace qmv
