"""GPU parity of the Q4_0 and Q5_K paths with the oracle.

FlareLLM：纯Rust打造的浏览器端LLM推理引擎, §量化技术的全面支持 names Q4_0 and the
K-quants among the formats read; the GGUF layouts are restated in include/qmv.h.
Blocks come from the synthetic generators and from the test-side encoder
(tests/blockpack.py) over each field's FULL range (fp16 scales of either sign,
subnormals, every quant value, scale and min 0..63), and every kernel that
serves these formats -- asserted through qmv_debug_last_kernel -- is compared
with the oracle element by element: dequantization bit for bit, matvecs within
|y - y_ref| <= 1e-4 * sum_i |w_i x_i| + 1e-6, the fused MoE step bit for bit
against the two-launch step, which is itself held to the oracle.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import quantized_decode_superblocks_b200 as q
from blockpack import pack_q4_0_many, pack_q5_k_many
from quantized_decode_superblocks_b200 import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

Q4_0, Q5_K = synth.Q4_0, synth.Q5_K
GEN, SK = q.KERNEL_GENERAL, q.KERNEL_STREAM
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
    """Finite fp16 scales of either sign: zero, subnormals and normals up to 2^4."""
    bits = (g.integers(0, 2, n) << 15) | (g.integers(0, 20, n) << 10) | g.integers(0, 1024, n)
    special = [0x0000, 0x8000, 0x0001, 0x83FF]
    bits[:min(n, 4)] = special[:min(n, 4)]
    return bits.astype(np.uint16)


def full_range_blocks(fmt, rows, cols, seed):
    g = np.random.default_rng(seed)
    n = rows * cols // synth.BLOCK_WEIGHTS[fmt]
    if fmt == Q4_0:
        qv = g.integers(0, 16, (n, 32))
        qv[n // 3, :] = 0
        qv[n // 2, :] = 15
        return pack_q4_0_many(fp16_bits(g, n), qv)
    sc, m = g.integers(0, 64, (n, 8)), g.integers(0, 64, (n, 8))
    sc[n // 3, :], m[n // 3, :] = 63, 63
    sc[n // 2, :], m[n // 2, :] = 0, 63
    sc[-1, :], m[-1, :] = 63, 0
    qv = g.integers(0, 32, (n, 256))
    qv[n // 3, :] = 31
    qv[-1, :] = 16                                    # fifth bits only
    return pack_q5_k_many(fp16_bits(g, n), fp16_bits(g, n), sc, m, qv)


def blocks(kind, fmt, rows, cols, seed):
    return full_range_blocks(fmt, rows, cols, seed) if kind == "full" else synth.gen_blocks(fmt, rows, cols,
                                                                                           seed, fmt)


def within(y, ref, bound):
    err = np.abs(np.asarray(y, np.float64) - ref)
    lim = REL * bound + ABS
    assert (err <= lim).all(), f"{(err > lim).sum()} outside tolerance, worst err/lim {(err / lim).max():.3g}"


def matvec(fmt, W, rows, cols, x):
    n_tok = x.shape[0]
    y = torch.full((n_tok, rows), float("nan"), device="cuda")
    if n_tok == 1:
        q.qmv_f32(fmt, dev(W), rows, cols, dev(x), y)
    else:
        q.qmv_batched(fmt, dev(W), rows, cols, dev(x), y, n_tok)
    kernel = q.qmv_debug_last_kernel()
    torch.cuda.synchronize()
    return y.cpu().numpy(), kernel


@pytest.mark.parametrize("kind", ["full", "synth"])
@pytest.mark.parametrize("fmt,rows,cols", [(Q4_0, 37, 96), (Q4_0, 300, 2048), (Q4_0, 3, 32),
                                           (Q5_K, 20, 768), (Q5_K, 300, 2048), (Q5_K, 1, 256)])
def test_dequant_bit_exact(kind, fmt, rows, cols):
    W = blocks(kind, fmt, rows, cols, 100 + rows)
    out = torch.full((rows, cols), float("nan"), device="cuda")
    q.qmv_dequant(fmt, dev(W), rows, cols, out)
    ref = oracle.dequant(fmt, W, rows, cols)
    assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))


# (fmt, rows, cols, n_tok, kernel that must serve the call)
PATHS = [
    (Q4_0, 300, 2048, 1, SK), (Q5_K, 300, 2048, 1, SK),          # streaming, one K-segment
    (Q4_0, 70, 8192, 1, SK), (Q5_K, 50, 8192, 1, SK),            # streaming, K-split rows
    (Q4_0, 46, 2176, 1, SK), (Q5_K, 45, 2304, 1, SK),            # a ragged last K-segment
    (Q4_0, 45, 2112, 1, GEN),                                    # row pairs not 16-byte multiples
    (Q4_0, 33, 12288, 1, SK), (Q5_K, 5, 12288, 1, SK),           # six K-segments
    (Q5_K, 3, 256, 1, SK), (Q5_K, 20, 768, 1, SK),               # fewer rows than a row slot
    (Q4_0, 37, 96, 1, GEN),                                      # rows not whole block pairs
    (Q4_0, 9, 32768, 1, GEN), (Q5_K, 9, 32768, 1, GEN),          # x beyond the streaming kernel's
    (Q4_0, 300, 2048, 2, SK), (Q5_K, 300, 2048, 2, SK),          # several tokens: streaming (2-4)
    (Q4_0, 300, 2048, 3, SK), (Q5_K, 37, 4096, 4, SK),
    (Q5_K, 300, 2048, 5, GEN),                                   # general (5-8)
    (Q4_0, 300, 2048, 8, GEN), (Q5_K, 300, 2048, 8, GEN),
    (Q4_0, 37, 96, 5, GEN), (Q5_K, 20, 768, 7, GEN),
    (Q4_0, 40, 16384, 4, GEN), (Q5_K, 40, 16384, 4, GEN),        # K-chunked rows
]


@pytest.mark.parametrize("kind", ["full", "synth"])
@pytest.mark.parametrize("fmt,rows,cols,n_tok,kernel", PATHS)
def test_matvec_every_path(kind, fmt, rows, cols, n_tok, kernel):
    W = blocks(kind, fmt, rows, cols, 2000 + 10 * fmt + n_tok)
    x = synth.gen_x(n_tok, cols, 2001, n_tok)
    y, k = matvec(fmt, W, rows, cols, x)
    assert k == kernel
    ref, bound = oracle.qmv(fmt, W, rows, cols, x, nthreads=8)
    within(y, ref, bound)


@pytest.mark.parametrize("fmt", [Q4_0, Q5_K])
def test_several_tokens_agree_with_single_token_calls(fmt):
    rows, cols = 257, 4096
    W = synth.gen_blocks(fmt, rows, cols, 31, fmt)
    x = synth.gen_x(8, cols, 31, 1)
    yb, _ = matvec(fmt, W, rows, cols, x)
    ref, bound = oracle.qmv(fmt, W, rows, cols, x)
    within(yb, ref, bound)
    for t in (0, 5, 7):
        y1, _ = matvec(fmt, W, rows, cols, x[t:t + 1])
        within(y1, ref[t:t + 1], bound[t:t + 1])


@pytest.mark.parametrize("fmt", [Q4_0, Q5_K])
@pytest.mark.parametrize("n_tok", [1, 4])
def test_grouped_launch(fmt, n_tok):
    shapes = [(300, 2048), (17, 4096), (5, 256)]
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


@pytest.mark.parametrize("fmt", [Q4_0, Q5_K])
def test_chain_dependent_tasks(fmt):
    dims = [2048, 4096, 2048, 6144, 2048]
    bufs = [dev(synth.gen_x(1, dims[0], 4001, 0)[0])] + [torch.full((d,), float("nan"), device="cuda")
                                                         for d in dims[1:]]
    Ws, args = [], []
    for t in range(len(dims) - 1):
        W = synth.gen_blocks(fmt, dims[t + 1], dims[t], 4000 + t, fmt)
        Ws.append(W)
        args.append((dev(W), dims[t + 1], dims[t], bufs[t], bufs[t + 1]))
    q.qmv_chain(fmt, args)
    assert q.qmv_debug_last_kernel() == SK
    torch.cuda.synchronize()
    outs = [b.cpu().numpy() for b in bufs]
    for t in range(len(dims) - 1):
        ref, bound = oracle.qmv(fmt, Ws[t], dims[t + 1], dims[t], outs[t][None, :])
        within(outs[t + 1][None, :], ref, bound)


@pytest.mark.parametrize("fmt,rows,cols,n_tok", [(Q5_K, 3000, 2048, 1), (Q4_0, 5000, 1024, 1),
                                                 (Q5_K, 777, 512, 4), (Q4_0, 300, 8192, 1)])
def test_argmax(fmt, rows, cols, n_tok):
    W = synth.gen_blocks(fmt, rows, cols, 40 + n_tok, fmt)
    x = synth.gen_x(n_tok, cols, 41, n_tok)
    yd = torch.full((n_tok, rows), float("nan"), device="cuda")
    idx = torch.full((n_tok,), -7, dtype=torch.int32, device="cuda")
    q.qmv_argmax(fmt, dev(W), rows, cols, dev(x), yd, n_tok, idx)
    if n_tok == 1 and cols <= 2048:
        assert q.qmv_debug_last_kernel() == SK          # fused into the streaming kernel's epilogue
    torch.cuda.synchronize()
    y, i = yd.cpu().numpy(), idx.cpu().numpy()
    ref, bound = oracle.qmv(fmt, W, rows, cols, x)
    within(y, ref, bound)
    for t in range(n_tok):
        assert i[t] == int(np.argmax(y[t]))


def _moe_check(fmt, gate, up, down, gus, ds, n_expert, ids, g32, hidden, inter, x, hh, yy):
    """h_k = silu(u_k) v_k with u_k, v_k each held to the single-matvec rule;
    y = sum_k g_k down_k h_k, fed the GPU's own h, to the same rule."""
    ref = oracle.moe_ffn(fmt, gate, up, gus, fmt, down, ds, n_expert, np.asarray(ids), g32.astype(np.float64),
                         hidden, inter, x)
    yref, bnd = np.zeros(hidden), np.zeros(hidden)
    for k, e in enumerate(ids):
        _, bu = oracle.qmv(fmt, gate[e * gus:(e + 1) * gus], inter, hidden, x)
        _, bv = oracle.qmv(fmt, up[e * gus:(e + 1) * gus], inter, hidden, x)
        du, dv = REL * bu[0] + ABS, REL * bv[0] + ABS
        u, v = ref["u"][k], ref["v"][k]
        su = u / (1 + np.exp(-u))
        dh = 1.1 * du * np.abs(v) + np.abs(su) * dv + 1.1 * du * dv + 1e-6 * np.abs(ref["h"][k])
        assert (np.abs(hh[k] - ref["h"][k]) <= dh + ABS).all(), k
        r, b = oracle.qmv(fmt, down[e * ds:(e + 1) * ds], hidden, inter, hh[k][None, :])
        yref += float(g32[k]) * r[0]
        bnd += abs(float(g32[k])) * b[0]
    within(yy[None, :], yref[None, :], bnd[None, :])


@pytest.mark.parametrize("fmt,n_expert,hidden,inter,top_k,kernel", [(Q5_K, 32, 2048, 1792, 4, SK),
                                                                    (Q4_0, 16, 1024, 512, 3, SK),
                                                                    (Q5_K, 8, 4096, 768, 6, SK),
                                                                    (Q4_0, 8, 512, 2304, 4, GEN)])
def test_moe_ffn_and_the_one_launch_step(fmt, n_expert, hidden, inter, top_k, kernel):
    seed = 90 + fmt
    gus, ds = synth.matrix_bytes(fmt, inter, hidden), synth.matrix_bytes(fmt, hidden, inter)
    gate = synth.gen_blocks(fmt, inter * n_expert, hidden, seed, 1)
    up = synth.gen_blocks(fmt, inter * n_expert, hidden, seed, 2)
    down = synth.gen_blocks(fmt, hidden * n_expert, inter, seed, 3)
    gd, ud, dd = dev(gate), dev(up), dev(down)
    ws = torch.zeros(q.MOE_WS_BYTES // 8, dtype=torch.int64, device="cuda")
    logits, bias = synth.gen_router(n_expert, seed, 5)
    lg, bs = dev(logits), dev(bias)
    x = synth.gen_x(1, hidden, seed, 4)[0]
    xd = dev(x)
    ids_a = torch.empty(top_k, dtype=torch.int32, device="cuda")
    g_a = torch.empty(top_k, device="cuda")
    h_a = torch.full((top_k, inter), float("nan"), device="cuda")
    y_a = torch.full((hidden,), float("nan"), device="cuda")
    q.moe_route(lg, bs, n_expert, top_k, ids_a, g_a)
    q.moe_ffn(fmt, gd, ud, gus, fmt, dd, ds, n_expert, ids_a, g_a, top_k, hidden, inter, xd, h_a, y_a)
    assert q.qmv_debug_last_kernel() == kernel
    torch.cuda.synchronize()
    ids = ids_a.cpu().tolist()
    _moe_check(fmt, gate, up, down, gus, ds, n_expert, ids, g_a.cpu().numpy(), hidden, inter, x,
               h_a.cpu().numpy(), y_a.cpu().numpy())
    # the one-launch step: the same ids, weights, h and y, bit for bit
    ids_b = torch.full((top_k,), -9, dtype=torch.int32, device="cuda")
    g_b = torch.full((top_k,), float("nan"), device="cuda")
    h_b = torch.full((top_k, inter), float("nan"), device="cuda")
    y_b = torch.full((hidden,), float("nan"), device="cuda")
    q.moe_ffn_routed(lg, bs, n_expert, top_k, fmt, gd, ud, gus, fmt, dd, ds, hidden, inter, xd,
                     ids_b, g_b, h_b, y_b, ws)
    assert q.qmv_debug_last_kernel() == kernel
    torch.cuda.synchronize()
    assert ids_b.cpu().tolist() == ids
    for a, b in ((g_a, g_b), (h_a, h_b), (y_a, y_b)):
        assert np.array_equal(a.cpu().numpy().view(np.uint32), b.cpu().numpy().view(np.uint32))


@pytest.mark.parametrize("fmt", [Q4_0, Q5_K])
def test_moe_qmv_weighted(fmt):
    n_expert, rows, cols = 6, 200, 2048
    mb = synth.matrix_bytes(fmt, rows, cols)
    E = full_range_blocks(fmt, rows * n_expert, cols, 5000 + fmt)
    ids = np.array([5, 0, 3], np.int32)
    x = synth.gen_x(1, cols, 5001, 0)
    gw = np.array([0.5, -0.25, 0.125], np.float32)
    y = torch.full((rows,), float("nan"), device="cuda")
    q.moe_qmv(fmt, dev(E), mb, n_expert, dev(ids), 3, rows, cols, dev(x), 0, dev(gw), y)
    assert q.qmv_debug_last_kernel() == GEN
    torch.cuda.synchronize()
    refs = [oracle.qmv(fmt, E[e * mb:(e + 1) * mb], rows, cols, x) for e in ids]
    within(y.cpu().numpy(), sum(float(gw[k]) * refs[k][0][0] for k in range(3)),
           sum(abs(float(gw[k])) * refs[k][1][0] for k in range(3)))
