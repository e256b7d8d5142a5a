"""Parity over the formats' FULL field ranges, through every kernel path.

The synthetic workloads draw fields from the configs' distributions, which
leave out values the formats allow: Q8_0 q = -128, Q6_K scales outside
[-64, 63], negative and subnormal fp16 scales.  Here every block is packed by
the test-side encoder (tests/blockpack.py) from fields drawn over the whole
range each field can hold (GGUF layouts as restated for BebeLM：纯Rust实现的端侧
大模型推理引擎, §量化格式支持), with the extremes forced into some blocks, and
each kernel path -- asserted through qmv_debug_last_kernel -- is compared with
the oracle element by element: dequantization bit for bit, matvecs within
|y - y_ref| <= 1e-4 * sum_i |w_i x_i| + 1e-6.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import quantized_decode_superblocks_b200 as q
from blockpack import pack_q4_k_many, pack_q6_k_many, pack_q8_0_many
from quantized_decode_superblocks_b200 import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

Q8_0, Q4_K, Q6_K = synth.Q8_0, synth.Q4_K, synth.Q6_K
WR, GEN, TC, SK = q.KERNEL_WARP_RING, q.KERNEL_GENERAL, q.KERNEL_TENSOR_CORE, q.KERNEL_STREAM
REL, ABS = 1e-4, 1e-6


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    q.build()
    q.lib()
    yield
    assert q.qmv_check() == 0


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def fp16_bits(g, n):
    """Finite fp16 scales of either sign: zero, subnormals and normals up to 2^4
    (exponent field 0..19), so no product overflows f32."""
    sign = g.integers(0, 2, n) << 15
    exp = g.integers(0, 20, n) << 10
    man = g.integers(0, 1024, n)
    bits = sign | exp | man
    bits[:4] = [0x0000, 0x8000, 0x0001, 0x83FF]       # +0, -0, smallest and largest negative subnormal
    return bits.astype(np.uint16)


def full_range_blocks(fmt, rows, cols, seed):
    g = np.random.default_rng(seed)
    n = rows * cols // synth.BLOCK_WEIGHTS[fmt]
    if fmt == Q8_0:
        qv = g.integers(-128, 128, (n, 32))
        qv[n // 3, :] = -128
        qv[n // 2, :] = 127
        return pack_q8_0_many(fp16_bits(g, n), qv)
    if fmt == Q4_K:
        sc, m = g.integers(0, 64, (n, 8)), g.integers(0, 64, (n, 8))
        sc[n // 3, :], m[n // 3, :] = 63, 63
        sc[n // 2, :], m[n // 2, :] = 0, 63
        sc[-1, :], m[-1, :] = 63, 0
        return pack_q4_k_many(fp16_bits(g, n), fp16_bits(g, n), sc, m, g.integers(0, 16, (n, 256)))
    s6 = g.integers(-128, 128, (n, 16))
    s6[n // 3, :] = -128
    s6[n // 2, :] = 127
    qv = g.integers(0, 64, (n, 256))
    qv[-1, :] = 0
    return pack_q6_k_many(fp16_bits(g, n), s6, qv)


def within(y, ref, bound):
    err = np.abs(np.asarray(y, np.float64) - ref)
    lim = REL * bound + ABS
    assert (err <= lim).all(), f"{(err > lim).sum()} outside tolerance, worst err/lim {(err / lim).max():.3g}"


def run(fmt, W, rows, cols, x, kernel):
    n_tok = x.shape[0]
    y = torch.full((n_tok, rows), float("nan"), device="cuda")
    if n_tok == 1:
        q.qmv_f32(fmt, dev(W), rows, cols, dev(x), y)
    else:
        q.qmv_batched(fmt, dev(W), rows, cols, dev(x), y, n_tok)
    assert q.qmv_debug_last_kernel() == kernel
    torch.cuda.synchronize()
    ref, bound = oracle.qmv(fmt, W, rows, cols, x, nthreads=8)
    within(y.cpu().numpy(), ref, bound)


@pytest.mark.parametrize("fmt,rows,cols", [(Q8_0, 37, 96), (Q8_0, 300, 2048), (Q4_K, 300, 2048),
                                           (Q6_K, 300, 2048), (Q6_K, 20, 768)])
def test_dequant_full_range_bit_exact(fmt, rows, cols):
    W = full_range_blocks(fmt, rows, cols, 1000 + fmt)
    out = torch.empty((rows, cols), device="cuda")
    q.qmv_dequant(fmt, dev(W), rows, cols, out)
    ref = oracle.dequant(fmt, W, rows, cols)
    assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))


# (fmt, rows, cols, n_tok, kernel that must serve the call)
PATHS = [
    (Q8_0, 300, 2048, 1, SK), (Q4_K, 300, 2048, 1, SK), (Q6_K, 300, 2048, 1, SK),     # streaming, one K-segment
    (Q8_0, 70, 8192, 1, SK), (Q6_K, 40, 4096, 1, SK), (Q4_K, 50, 8192, 1, SK),        # streaming, K-split rows
    (Q6_K, 24, 1792, 1, GEN),                                                          # rows not 16-byte multiples
    (Q8_0, 33, 12288, 1, SK), (Q6_K, 8, 10240, 1, SK),                                 # streaming, 6 / 5 K-segments
    (Q4_K, 5, 12288, 1, SK), (Q8_0, 37, 96, 1, GEN),                                   # 6 K-segments; general
    (Q8_0, 300, 2048, 2, SK), (Q4_K, 300, 2048, 2, SK), (Q6_K, 300, 2048, 2, SK),     # streaming, two tokens
    (Q8_0, 70, 8192, 2, SK), (Q4_K, 9, 12288, 2, SK), (Q6_K, 36, 1024, 3, SK),       # K-split rows; Q6_K 3 tokens
    (Q6_K, 300, 8192, 4, WR),                                                          # warp-ring: 128 KB of x
    (Q8_0, 300, 2048, 3, TC), (Q4_K, 300, 2048, 3, TC), (Q6_K, 300, 2048, 3, TC),     # tensor cores
    (Q8_0, 300, 2048, 8, TC), (Q4_K, 300, 2048, 8, TC), (Q6_K, 300, 2048, 8, TC),
    (Q4_K, 9, 512, 5, TC),                                                             # a partial tensor-core tile
    (Q8_0, 37, 96, 5, GEN), (Q6_K, 20, 768, 8, GEN),                                  # general, several tokens
]


@pytest.mark.parametrize("fmt,rows,cols,n_tok,kernel", PATHS)
def test_matvec_full_range_every_path(fmt, rows, cols, n_tok, kernel):
    W = full_range_blocks(fmt, rows, cols, 2000 + 10 * fmt + n_tok)
    x = synth.gen_x(n_tok, cols, 2001, n_tok)
    run(fmt, W, rows, cols, x, kernel)


@pytest.mark.parametrize("fmt", [Q8_0, Q4_K, Q6_K])
@pytest.mark.parametrize("n_tok", [1, 4])
def test_grouped_launch_full_range(fmt, n_tok):
    shapes = [(300, 2048), (17, 4096), (5, 256 if fmt != Q8_0 else 64)]
    host, args = [], []
    for i, (rows, cols) in enumerate(shapes):
        W = full_range_blocks(fmt, rows, cols, 3000 + 10 * fmt + i)
        x = synth.gen_x(n_tok, cols, 3001, i)
        y = torch.full((n_tok, rows), float("nan"), device="cuda")
        host.append((W, rows, cols, x))
        args.append((dev(W), rows, cols, dev(x), y))
    q.qmv_multi(fmt, n_tok, args)
    assert q.qmv_debug_last_kernel() == GEN
    torch.cuda.synchronize()
    for (W, rows, cols, x), a in zip(host, args):
        ref, bound = oracle.qmv(fmt, W, rows, cols, x)
        within(a[4].cpu().numpy(), ref, bound)


@pytest.mark.parametrize("fmt", [Q8_0, Q6_K])
def test_chain_full_range(fmt):
    dims = [2048, 4096, 2048]           # every row a multiple of 16 bytes: the persistent kernel takes it
    bufs = [dev(synth.gen_x(1, dims[0], 4001, 0)[0])] + [torch.full((d,), float("nan"), device="cuda")
                                                         for d in dims[1:]]
    Ws, args = [], []
    for t in range(len(dims) - 1):
        W = full_range_blocks(fmt, dims[t + 1], dims[t], 4000 + t)
        Ws.append(W)
        args.append((dev(W), dims[t + 1], dims[t], bufs[t], bufs[t + 1]))
    q.qmv_chain(fmt, args)
    assert q.qmv_debug_last_kernel() == SK
    torch.cuda.synchronize()
    outs = [b.cpu().numpy() for b in bufs]
    for t in range(len(dims) - 1):
        ref, bound = oracle.qmv(fmt, Ws[t], dims[t + 1], dims[t], outs[t][None, :])
        within(outs[t + 1][None, :], ref, bound)


def test_moe_weighted_full_range_q8_0():
    n_expert, rows, cols = 6, 200, 2048
    mb = synth.matrix_bytes(Q8_0, rows, cols)
    E = full_range_blocks(Q8_0, rows * n_expert, cols, 5000)
    ids = np.array([5, 0, 3], np.int32)
    x = synth.gen_x(1, cols, 5001, 0)
    gw = np.array([0.5, -0.25, 0.125], np.float32)
    y = torch.full((rows,), float("nan"), device="cuda")
    q.moe_qmv(Q8_0, dev(E), mb, n_expert, dev(ids), 3, rows, cols, dev(x), 0, dev(gw), y)
    assert q.qmv_debug_last_kernel() == GEN
    torch.cuda.synchronize()
    refs = [oracle.qmv(Q8_0, E[e * mb:(e + 1) * mb], rows, cols, x) for e in ids]
    within(y.cpu().numpy(), sum(float(gw[k]) * refs[k][0][0] for k in range(3)),
           sum(abs(float(gw[k])) * refs[k][1][0] for k in range(3)))
