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

enum { FMT_Q8_0 = 0, FMT_Q4_K = 1, FMT_Q6_K = 2, FMT_Q4_0 = 3, FMT_Q5_K = 4 };

template <int FMT> struct Fmt;
template <> struct Fmt<FMT_Q8_0> { static constexpr int BW = 32;  static constexpr int BB = 34; };
template <> struct Fmt<FMT_Q4_K> { static constexpr int BW = 256; static constexpr int BB = 144; };
template <> struct Fmt<FMT_Q6_K> { static constexpr int BW = 256; static constexpr int BB = 210; };
template <> struct Fmt<FMT_Q4_0> { static constexpr int BW = 32;  static constexpr int BB = 18; };
template <> struct Fmt<FMT_Q5_K> { static constexpr int BW = 256; static constexpr int BB = 176; };

// Formats whose one-token slice is one 32-weight block (else 64 weights of a
// 256-weight superblock), and the K-quants that share Q4_K's scale packing.
template <int FMT> constexpr bool small_block() { return FMT == FMT_Q8_0 || FMT == FMT_Q4_0; }
template <int FMT> constexpr bool q4k_like() { return FMT == FMT_Q4_K || FMT == FMT_Q5_K; }

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

__device__ __forceinline__ float4 lds_f4(uint32_t a)
{
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a));
    return v;
}

__device__ __forceinline__ uint2 lds_v2(uint32_t a)
{
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}

__device__ __forceinline__ float2 lds_f2(uint32_t a)
{
    float2 v;
    asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(a));
    return v;
}

__device__ __forceinline__ void sts_f4(uint32_t a, float4 v)
{
    asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};"
                 :: "r"(a), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w) : "memory");
}

__device__ __forceinline__ void sts_v4(uint32_t a, uint4 v)
{
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" :: "r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
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

#ifndef QMV_WAIT_MODE
#define QMV_WAIT_MODE 1
#endif
// One poll of the phase with the given parity.  Mode 0: blocking try_wait with
// the system's suspend window; mode 1: try_wait with a short suspend hint, so a
// warp that went to sleep on a not-yet-landed stage wakes up promptly; mode 2:
// non-blocking test_wait.
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
#if QMV_WAIT_MODE == 0
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
#elif QMV_WAIT_MODE == 1
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(bar), "r"(parity), "r"(200u) : "memory");
#else
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
#endif
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

// As mbar_wait_bounded, polling with the blocking try_wait and no suspend-time
// hint: the thread sleeps until the phase completes or the system's time
// window ends.  Measured faster than the hinted form for the streaming
// kernel, whose consumer warps often wait on data in flight.
__device__ __forceinline__ bool mbar_wait_bounded_block(uint32_t bar, uint32_t parity)
{
    auto poll = [&]() {
        uint32_t ok;
        asm volatile("{\n\t.reg .pred p;\n\t"
                     "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                     "selp.u32 %0, 1, 0, p;\n\t}"
                     : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
        return ok != 0;
    };
    if (poll()) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t i = 1;; ++i) {
        if (poll()) return true;
        if ((i & 15u) == 0u && global_timer_ns() - t0 > 1000000000ull) return false;
    }
}

// One 1-D bulk copy global -> this CTA's shared memory, completing on `bar`.
// dst, src 16-byte aligned, bytes a multiple of 16.  Local memory only.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 :: "r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}

// An L2 policy that evicts the lines it tags first: for weights, which a
// decode step reads once, so that streaming them does not push the
// activations and the kernels' code out of L2.
__device__ __forceinline__ uint64_t l2_evict_first_policy()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// bulk_g2s with an L2 cache policy (l2_evict_first_policy).
__device__ __forceinline__ void bulk_g2s_hint(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar,
                                              uint64_t pol)
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

// ------------------------------------------------------- greedy argmax --
// Candidate (value, row) pairs: IEEE > on f32, ties to the lower row; bi < 0
// means no candidate.  A 64-bit key orders candidates the same way: the
// value's bits mapped to an order-preserving unsigned in the high word, the
// complement of the row in the low word, so an atomic max over keys picks the
// same winner in any order.
__device__ __forceinline__ void argmax_merge(float &bv, int &bi, float ov, int oi)
{
    if (oi < 0) return;
    if (bi < 0 || ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
    }
}

__device__ __forceinline__ unsigned long long argmax_key(float v, int row)
{
    const uint32_t u = v == 0.f ? 0u : __float_as_uint(v);            // -0 and +0 compare equal
    const uint32_t hi = (u & 0x80000000u) ? ~u : (u | 0x80000000u);   // order-preserving for non-NaN
    return ((unsigned long long)hi << 32) | (uint32_t)(0xFFFFFFFFu - (uint32_t)row);
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
