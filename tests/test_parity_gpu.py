"""Parity of the CUDA path (through the C ABI) with the oracle.

Bars: dequantization bit-exact; every matvec output within
|y - y_ref| <= 1e-4 * sum_i |w_i x_i| + 1e-6 (y_ref, the bound: f64 oracle);
router ids exact (a margin at the top-k cut is asserted first), weights within
1e-6 relative; the MoE FFN by the composite rule written in each test.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import quantized_decode_superblocks_b200 as q
from quantized_decode_superblocks_b200 import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

Q8_0, Q4_K, Q6_K = synth.Q8_0, synth.Q4_K, synth.Q6_K
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


def within(y, ref, bound, rel=REL, abs_=ABS):
    y = np.asarray(y, dtype=np.float64)
    err = np.abs(y - ref)
    lim = rel * bound + abs_
    bad = err > lim
    assert not bad.any(), (f"{bad.sum()} of {bad.size} outside tolerance; worst err/lim "
                           f"{(err / lim).max():.3g} at {np.unravel_index((err / lim).argmax(), err.shape)}")
    return float((err / lim).max())


def run_qmv(fmt, W, rows, cols, x):
    x = np.atleast_2d(x)
    n_tok = x.shape[0]
    Wd, xd = dev(W), dev(x)
    yd = torch.full((n_tok, rows), float("nan"), device="cuda")
    if n_tok == 1:
        q.qmv_f32(fmt, Wd, rows, cols, xd, yd)
    else:
        q.qmv_batched(fmt, Wd, rows, cols, xd, yd, n_tok)
    torch.cuda.synchronize()
    return yd.cpu().numpy()


# ----------------------------------------------------------------- dequant --

@pytest.mark.parametrize("fmt,rows,cols", [(Q8_0, 37, 96), (Q8_0, 5, 2048), (Q4_K, 37, 512),
                                           (Q4_K, 3, 1792), (Q6_K, 37, 768), (Q6_K, 2, 2048)])
def test_dequant_bit_exact(fmt, rows, cols):
    W = synth.gen_blocks(fmt, rows, cols, seed=31, tensor_id=fmt)
    out = torch.empty((rows, cols), device="cuda")
    q.qmv_dequant(fmt, dev(W), rows, cols, out)
    ref = oracle.dequant(fmt, W, rows, cols)
    assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))


def test_fp16_decode_every_pattern_on_gpu():
    # one Q8_0 block per fp16 pattern: d = pattern, q[0] = 1  ->  w[0] = f32(d)
    n = 65536
    W = np.zeros((n, 34), np.uint8)
    W[:, 0] = np.arange(n) & 0xFF
    W[:, 1] = np.arange(n) >> 8
    W[:, 2] = 1
    out = torch.empty((n, 32), device="cuda")
    q.qmv_dequant(Q8_0, dev(W.reshape(-1)), n, 32, out)
    got = out[:, 0].cpu().numpy()
    ref = np.array([oracle.half_to_float(b) for b in range(n)], np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_dequant_rejects_with_status_and_leaves_output():
    out = torch.full((4, 256), 7.0, device="cuda")
    with pytest.raises(q.QmvError):
        q.qmv_dequant(Q4_K, dev(np.zeros(4 * 144, np.uint8)), 4, 200, out)
    assert bool((out == 7.0).all())


# ------------------------------------------------------------------ matvec --

SMALL = [
    (Q8_0, 1, 32), (Q8_0, 3, 96), (Q8_0, 37, 1024), (Q8_0, 257, 2048), (Q8_0, 70, 4096),
    (Q4_K, 1, 256), (Q4_K, 3, 512), (Q4_K, 37, 1792), (Q4_K, 257, 2048), (Q4_K, 20, 4096),
    (Q6_K, 1, 256), (Q6_K, 3, 768), (Q6_K, 37, 1792), (Q6_K, 257, 2048), (Q6_K, 20, 4096),
]


@pytest.mark.parametrize("fmt,rows,cols", SMALL)
@pytest.mark.parametrize("n_tok", [1, 2, 3, 5, 8])
def test_qmv_small_shapes(fmt, rows, cols, n_tok):
    W = synth.gen_blocks(fmt, rows, cols, seed=7, tensor_id=100 + fmt)
    x = synth.gen_x(n_tok, cols, seed=7, tensor_id=200 + n_tok)
    y = run_qmv(fmt, W, rows, cols, x)
    ref, bound = oracle.qmv(fmt, W, rows, cols, x)
    within(y, ref, bound)


# Small one-token matrices: when a CTA's share of rows fills at most half of
# one stage the streaming kernel takes fewer rows per warp (Q4_K 3072x2048:
# 2 instead of 4; 700 rows: 1); Q8_0 1000x128 prefers one row per warp, whose
# 136-byte copies are not 16-byte multiples, and falls back to two.  The
# streaming kernel must serve every case.
@pytest.mark.parametrize("fmt,rows,cols", [(Q4_K, 3072, 2048), (Q4_K, 700, 2048), (Q8_0, 1024, 1024),
                                           (Q8_0, 1000, 128), (Q6_K, 500, 2048), (Q8_0, 148 * 12 + 5, 2048),
                                           (Q4_K, 148 * 24 + 3, 2048)])
def test_small_matrices_rows_per_warp(fmt, rows, cols):
    W = synth.gen_blocks(fmt, rows, cols, seed=31, tensor_id=rows)
    x = synth.gen_x(1, cols, seed=31, tensor_id=cols)
    y = run_qmv(fmt, W, rows, cols, x)
    assert q.qmv_debug_last_kernel() == q.KERNEL_STREAM
    ref, bound = oracle.qmv(fmt, W, rows, cols, x)
    within(y, ref, bound)


@pytest.mark.parametrize("fmt,rows,cols", [(Q8_0, 300, 8192), (Q8_0, 9, 16384), (Q4_K, 40, 16384),
                                           (Q6_K, 33, 8192), (Q8_0, 17, 8224), (Q6_K, 5, 4352),
                                           (Q8_0, 5, 65536), (Q4_K, 3, 65536), (Q6_K, 4, 34816),
                                           (Q8_0, 2, 40992)])
@pytest.mark.parametrize("n_tok", [1, 4, 8])
def test_qmv_long_rows_k_chunked(fmt, rows, cols, n_tok):
    W = synth.gen_blocks(fmt, rows, cols, seed=8, tensor_id=300 + fmt)
    x = synth.gen_x(n_tok, cols, seed=8, tensor_id=400 + n_tok)
    y = run_qmv(fmt, W, rows, cols, x)
    ref, bound = oracle.qmv(fmt, W, rows, cols, x)
    within(y, ref, bound)


# Q8_0 and Q4_K with 3..8 tokens and rows of whole 256-column K-chunks take
# the tensor-core kernel: partial row tiles, more tiles than CTAs, every
# K-split (1, 2, 4, 8 warps per tile), x in shared memory and through L2, and
# x over a wide range of magnitudes (the hi / lo bf16 split of x).
@pytest.mark.parametrize("fmt", [Q8_0, Q4_K])
@pytest.mark.parametrize("rows,cols", [(5, 256), (16, 768), (33, 512), (2371, 1024), (300, 2048),
                                       (16 * 148 * 2 + 7, 2048), (40, 8192)])
@pytest.mark.parametrize("n_tok", [3, 4, 6, 7, 8])
def test_tensor_core_tiles(fmt, rows, cols, n_tok):
    W = synth.gen_blocks(fmt, rows, cols, seed=11, tensor_id=rows)
    x = synth.gen_x(n_tok, cols, seed=11, tensor_id=cols + n_tok)
    y = run_qmv(fmt, W, rows, cols, x)
    ref, bound = oracle.qmv(fmt, W, rows, cols, x, nthreads=8)
    within(y, ref, bound)


# Q6_K takes it when rows are whole 2048-column runs and every token's x fits
# in shared memory beside two-stage rings: superblocks at every 2-byte offset
# within their 16-byte-aligned slots, the last row's copy cut at the end of the
# matrix.  The kernel that served each case is asserted; 8 tokens of 4096
# columns (131 KB of split x) do not fit and take the general kernel.
@pytest.mark.parametrize("rows,cols,n_tok,kernel", [
    (5, 2048, 3, q.KERNEL_TENSOR_CORE), (5, 2048, 4, q.KERNEL_TENSOR_CORE), (5, 2048, 8, q.KERNEL_TENSOR_CORE),
    (16 * 148 * 2 + 7, 2048, 3, q.KERNEL_TENSOR_CORE), (16 * 148 * 2 + 7, 2048, 8, q.KERNEL_TENSOR_CORE),
    (300, 4096, 3, q.KERNEL_TENSOR_CORE), (300, 4096, 4, q.KERNEL_TENSOR_CORE), (16, 6144, 3, q.KERNEL_TENSOR_CORE),
    (300, 4096, 8, q.KERNEL_GENERAL)])
def test_tensor_core_q6_k_tiles(rows, cols, n_tok, kernel):
    W = synth.gen_blocks(Q6_K, rows, cols, seed=14, tensor_id=rows)
    x = synth.gen_x(n_tok, cols, seed=14, tensor_id=cols + n_tok)
    y = run_qmv(Q6_K, W, rows, cols, x)
    assert q.qmv_debug_last_kernel() == kernel
    ref, bound = oracle.qmv(Q6_K, W, rows, cols, x, nthreads=8)
    within(y, ref, bound)


@pytest.mark.parametrize("fmt", [Q8_0, Q4_K, Q6_K])
@pytest.mark.parametrize("scale", [1e-30, 1e-6, 1e6, 1e30])
def test_tensor_core_x_magnitudes(fmt, scale):
    rows, cols, n_tok = 64, 2048, 8
    W = synth.gen_blocks(fmt, rows, cols, seed=12, tensor_id=0)
    x = (synth.gen_x(n_tok, cols, seed=12, tensor_id=1) * np.float32(scale)).astype(np.float32)
    y = run_qmv(fmt, W, rows, cols, x)
    ref, bound = oracle.qmv(fmt, W, rows, cols, x)
    within(y, ref, bound, abs_=ABS * min(1.0, scale))


@pytest.mark.parametrize("fmt", [Q8_0, Q4_K, Q6_K])
def test_tensor_core_repeatable(fmt):
    # the K-split partial sums are added in a fixed order: identical bits every call
    rows, cols, n_tok = 3072, 2048, 8
    W = synth.gen_blocks(fmt, rows, cols, seed=13, tensor_id=0)
    x = synth.gen_x(n_tok, cols, seed=13, tensor_id=1)
    a = run_qmv(fmt, W, rows, cols, x)
    b = run_qmv(fmt, W, rows, cols, x)
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))


@pytest.mark.parametrize("n_tok", [1, 4, 8])
def test_every_n_tok_agrees_with_single_token_calls(n_tok):
    fmt, rows, cols = Q6_K, 129, 2048
    W = synth.gen_blocks(fmt, rows, cols, seed=9, tensor_id=1)
    x = synth.gen_x(n_tok, cols, seed=9, tensor_id=2)
    yb = run_qmv(fmt, W, rows, cols, x)
    ref, bound = oracle.qmv(fmt, W, rows, cols, x)
    for t in range(n_tok):
        within(run_qmv(fmt, W, rows, cols, x[t]), ref[t:t + 1], bound[t:t + 1])
    within(yb, ref, bound)


def test_closed_form_constant_blocks_on_gpu():
    # Q4_K with every field constant: y = (d*S*Q - dmin*M) * sum(x) for every row
    from blockpack import f16_bits, pack_q4_k, pack_q8_0
    d, dmin, S, Q, M = 0.0078125, 0.00390625, 37, 11, 5
    rows, cols = 64, 2048
    blk = pack_q4_k(f16_bits(d), f16_bits(dmin), [S] * 8, [M] * 8, [Q] * 256)
    x = synth.gen_x(1, cols, 13, 0)
    y = run_qmv(Q4_K, np.tile(blk, rows * cols // 256), rows, cols, x)
    exact = (d * S * Q - dmin * M) * float(np.sum(x.astype(np.float64)))
    bound = (abs(d * S * Q - dmin * M)) * float(np.sum(np.abs(x.astype(np.float64))))
    within(y, np.full_like(y, exact, dtype=np.float64), np.full(y.shape, bound))
    # Q8_0 with d = 1 and small integer x: the dot is an exact integer
    g = np.random.default_rng(5)
    qv = g.integers(-127, 128, size=(8, 1024))
    W8 = np.concatenate([pack_q8_0(f16_bits(1.0), qv[r, 32 * b:32 * b + 32])
                         for r in range(8) for b in range(32)])
    xi = g.integers(-8, 9, size=(1, 1024)).astype(np.float32)
    y8 = run_qmv(Q8_0, W8, 8, 1024, xi)
    assert y8[0].tolist() == [float(v) for v in (qv @ xi[0].astype(np.int64))]


def test_results_are_deterministic():
    fmt, rows, cols = Q4_K, 3072, 2048
    W = synth.gen_blocks(fmt, rows, cols, seed=1, tensor_id=0)
    x = synth.gen_x(1, cols, seed=1, tensor_id=1)
    ys = [run_qmv(fmt, W, rows, cols, x) for _ in range(5)]
    for y in ys[1:]:
        assert np.array_equal(y.view(np.uint32), ys[0].view(np.uint32))


# ------------------------------------------------------- grouped launch --

@pytest.mark.parametrize("fmt,n_tok", [(Q8_0, 1), (Q4_K, 1), (Q6_K, 1), (Q8_0, 4), (Q4_K, 8)])
def test_qmv_multi_matches_each_task(fmt, n_tok):
    bw = synth.BLOCK_WEIGHTS[fmt]
    shapes = [(3072, 2048), (2048, 2048), (257, 4096), (1, bw), (5000, 1792 if fmt == Q8_0 else 2048),
              (300, 8192), (17, 16384 if fmt != Q6_K else 8192), (1024, 1024 if fmt == Q8_0 else 2048)]
    host, dev_args = [], []
    for i, (rows, cols) in enumerate(shapes):
        W = synth.gen_blocks(fmt, rows, cols, 60 + fmt, i)
        x = synth.gen_x(n_tok, cols, 61, i)
        y = torch.full((n_tok, rows), float("nan"), device="cuda")
        host.append((W, rows, cols, x))
        dev_args.append((dev(W), rows, cols, dev(x), y))
    q.qmv_multi(fmt, n_tok, dev_args)
    torch.cuda.synchronize()
    for (W, rows, cols, x), (_, _, _, _, y) in zip(host, dev_args):
        ref, bound = oracle.qmv(fmt, W, rows, cols, x)
        within(y.cpu().numpy(), ref, bound)


def test_qmv_multi_many_tasks_and_errors():
    # more tasks than one launch takes, all from one shared weight matrix
    fmt, rows, cols = Q4_K, 96, 512
    W = synth.gen_blocks(fmt, rows, cols, 70, 0)
    Wd = dev(W)
    xs = synth.gen_x(130, cols, 70, 1)
    xd = dev(xs)
    y = torch.full((130, rows), float("nan"), device="cuda")
    tasks = [(Wd, rows, cols, xd[i], y[i]) for i in range(130)]
    q.qmv_multi(fmt, 1, tasks)
    torch.cuda.synchronize()
    ref, bound = oracle.qmv(fmt, W, rows, cols, xs)
    within(y.cpu().numpy(), ref, bound)
    with pytest.raises(q.QmvError):
        q.qmv_multi(fmt, 1, [(Wd, rows, 100, xd[0], y[0])])
    with pytest.raises(q.QmvError):
        q.qmv_multi(fmt, 9, tasks[:2])


# ------------------------------------------------------- chained launch --

def _chain_case(fmt, dims, seed):
    """Tasks t = 0..len(dims)-2 with W_t of shape dims[t+1] x dims[t]; task t
    reads task t-1's output as x (task 0 reads a fresh x).  Outputs start as NaN,
    so a task that ran before its input was complete would be caught."""
    Ws, dev_args = [], []
    x0 = synth.gen_x(1, dims[0], seed, 99)[0]
    bufs = [dev(x0)] + [torch.full((d,), float("nan"), device="cuda") for d in dims[1:]]
    for t in range(len(dims) - 1):
        cols, rows = dims[t], dims[t + 1]
        W = synth.gen_blocks(fmt, rows, cols, seed, t)
        Wd = dev(W)
        Ws.append((W, Wd))
        dev_args.append((Wd, rows, cols, bufs[t], bufs[t + 1]))
    q.qmv_chain(fmt, dev_args)
    torch.cuda.synchronize()
    outs = [b.cpu().numpy() for b in bufs]
    worst = 0.0
    for t in range(len(dims) - 1):
        # each step against the oracle on the input the GPU actually had
        ref, bound = oracle.qmv(fmt, Ws[t][0], dims[t + 1], dims[t], outs[t][None, :])
        worst = max(worst, within(outs[t + 1][None, :], ref, bound))
    return worst


@pytest.mark.parametrize("fmt", [Q8_0, Q4_K, Q6_K])
def test_qmv_chain_dependent_tasks(fmt):
    # x of every task is the previous task's y: the launches must be ordered
    dims = [2048, 3072, 2048, 16384, 2048, 8192, 2048] if fmt != Q6_K else [2048, 4096, 2048, 6144, 2048]
    _chain_case(fmt, dims, 80 + fmt)


def test_qmv_chain_long():
    # 70 tasks on 512 x 512 Q4_K matrices; task t reads task t-1's output
    # unless t % 3 == 0 (then a fresh x), so activations stay finite
    fmt, n, T = Q4_K, 512, 70
    x0 = synth.gen_x(1, n, 93, 0)[0]
    x0d = dev(x0)
    ys = torch.full((T, n), float("nan"), device="cuda")
    Ws, args = [], []
    for t in range(T):
        W = synth.gen_blocks(fmt, n, n, 93, 1 + t)
        Wd = dev(W)
        Ws.append(W)
        args.append((Wd, n, n, x0d if t % 3 == 0 else ys[t - 1], ys[t]))
    q.qmv_chain(fmt, args)
    torch.cuda.synchronize()
    yh = ys.cpu().numpy()
    for t in range(T):
        xin = x0 if t % 3 == 0 else yh[t - 1]
        ref, bound = oracle.qmv(fmt, Ws[t], n, n, xin[None, :])
        within(yh[t][None, :], ref, bound)


def test_qmv_chain_fallback_shape_keeps_order():
    # 96 columns is not a whole number of Q8_0 block pairs: one launch per task
    dims = [1024, 96, 2048, 1024]
    _chain_case(Q8_0, dims, 91)


def test_qmv_chain_repeated_calls():
    for rep in range(3):
        _chain_case(Q8_0, [1024, 2048, 512, 1024], 92 + rep)


def test_qmv_chain_on_two_streams_at_once():
    # the call keeps no state between calls: two chains may overlap
    dims = [2048, 4096, 2048, 8192, 2048]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    cases = []
    for s_i, st in enumerate(streams):
        bufs = [dev(synth.gen_x(1, dims[0], 94 + s_i, 0)[0])] + [torch.full((d,), float("nan"), device="cuda")
                                                                 for d in dims[1:]]
        Ws = [synth.gen_blocks(Q8_0, dims[t + 1], dims[t], 94 + s_i, t) for t in range(len(dims) - 1)]
        args = [(dev(W), dims[t + 1], dims[t], bufs[t], bufs[t + 1]) for t, W in enumerate(Ws)]
        cases.append((st, bufs, Ws, args))
    torch.cuda.synchronize()
    for st, _, _, args in cases:
        q.qmv_chain(Q8_0, args, st)
    torch.cuda.synchronize()
    for _, bufs, Ws, _ in cases:
        outs = [b.cpu().numpy() for b in bufs]
        for t in range(len(dims) - 1):
            ref, bound = oracle.qmv(Q8_0, Ws[t], dims[t + 1], dims[t], outs[t][None, :])
            within(outs[t + 1][None, :], ref, bound)


# ------------------------------------------------------------ greedy argmax --

def _argmax_check(fmt, W, rows, cols, x, seed_note=""):
    n_tok = x.shape[0]
    yd = torch.full((n_tok, rows), float("nan"), device="cuda")
    idx = torch.full((n_tok,), -7, dtype=torch.int32, device="cuda")
    q.qmv_argmax(fmt, dev(W), rows, cols, dev(x), yd, n_tok, idx)
    torch.cuda.synchronize()
    y, i = yd.cpu().numpy(), idx.cpu().numpy()
    ref, bound = oracle.qmv(fmt, W, rows, cols, x)
    within(y, ref, bound)
    for t in range(n_tok):
        # exact: the first maximum of the GPU's own logits (numpy's tie rule)
        assert i[t] == int(np.argmax(y[t])), (t, i[t], int(np.argmax(y[t])))
        # against the oracle: equal where the top two are further apart than
        # the error allowed on either; else the pick must be a near-maximum
        r = ref[t]
        lim = REL * bound[t] + ABS
        order = np.argsort(r, kind="stable")
        top = int(np.argmax(r))
        clear = rows == 1 or r[top] - r[order[-2]] > lim[top] + lim[order[-2]]
        if clear:
            assert i[t] == top
        else:
            assert r[i[t]] >= r[top] - 2 * lim.max()
    return i


@pytest.mark.parametrize("fmt,rows,cols,n_tok", [(Q6_K, 128000, 2048, 1), (Q6_K, 128000, 2048, 4),
                                                 (Q8_0, 5000, 1024, 1), (Q4_K, 777, 512, 8),
                                                 (Q4_K, 3000, 2048, 1), (Q8_0, 300, 8192, 1)])
def test_argmax_matches_logits_and_oracle(fmt, rows, cols, n_tok):
    W = synth.gen_blocks(fmt, rows, cols, 40 + n_tok, fmt)
    x = synth.gen_x(n_tok, cols, 41, n_tok)
    _argmax_check(fmt, W, rows, cols, x)
    # one token on rows of <= 2048 columns: fused into the streaming kernel's epilogue
    if n_tok == 1 and cols <= 2048:
        assert q.qmv_debug_last_kernel() == q.KERNEL_STREAM


def test_argmax_workspaces_on_two_streams():
    # two argmax calls in flight at once on two streams, each with its own
    # workspace: both choices correct, workspaces back to zero
    shapes = [(Q6_K, 64000, 2048, 60), (Q8_0, 70000, 2048, 61)]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    ws = [torch.zeros(q.ARGMAX_WS_BYTES // 8, dtype=torch.int64, device="cuda") for _ in range(2)]
    data = []
    for fmt, rows, cols, seed in shapes:
        W = synth.gen_blocks(fmt, rows, cols, seed, 0)
        x = synth.gen_x(1, cols, seed, 1)
        data.append((fmt, W, rows, cols, x, dev(W), dev(x), torch.empty((1, rows), device="cuda"),
                     torch.full((1,), -7, dtype=torch.int32, device="cuda")))
    torch.cuda.synchronize()
    for rep in range(3):
        for k, (fmt, W, rows, cols, x, Wd, xd, yd, idx) in enumerate(data):
            q.qmv_argmax_ws(fmt, Wd, rows, cols, xd, yd, 1, idx, ws[k], streams[k])
    torch.cuda.synchronize()
    for k, (fmt, W, rows, cols, x, Wd, xd, yd, idx) in enumerate(data):
        y = yd.cpu().numpy()
        assert int(idx.cpu()[0]) == int(np.argmax(y[0]))
        ref, bound = oracle.qmv_rows(fmt, W, rows, cols, np.array([int(idx.cpu()[0])]), x)
        within(y[:, [int(idx.cpu()[0])]], ref, bound)
        assert int(ws[k].abs().sum().cpu()) == 0


def test_argmax_ties_go_to_the_lower_row_and_nan_is_skipped():
    # rows of zero blocks (d = 0: logit 0) and three copies of one row with a
    # positive logit at rows 5, 9 and 14: bit-identical maxima, row 5 wins
    fmt, cols, rows = Q8_0, 256, 16
    one = synth.gen_blocks(fmt, 1, cols, 50, 0)
    x = synth.gen_x(1, cols, 53, 0)
    if oracle.qmv(fmt, one, 1, cols, x)[0][0, 0] < 0:
        x = -x
    W = np.zeros((rows, one.size), np.uint8)
    for r in (5, 9, 14):
        W[r] = one
    i = _argmax_check(fmt, W.reshape(-1), rows, cols, x)
    assert i[0] == 5
    # every row the same: row 0
    i = _argmax_check(fmt, np.tile(one, rows), rows, cols, x)
    assert i[0] == 0
    # a NaN activation makes every logit NaN: no row is chosen
    xn = x.copy()
    xn[0, 3] = np.nan
    yd = torch.empty((1, rows), device="cuda")
    idx = torch.zeros(1, dtype=torch.int32, device="cuda")
    q.qmv_argmax(fmt, dev(W), rows, cols, dev(xn), yd, 1, idx)
    torch.cuda.synchronize()
    assert np.isnan(yd.cpu().numpy()).all() and int(idx.cpu()[0]) == -1


# ---------------------------------------------------- full-size workloads --

def test_cfg0_q8_0_1024x1024():
    w = synth.workload_cfg0()
    W = synth.gen_blocks(w["fmt"], w["rows"], w["cols"], w["seed"], 0)
    x = synth.gen_x(1, w["cols"], w["seed"], 1)
    y = run_qmv(w["fmt"], W, w["rows"], w["cols"], x)
    ref, bound = oracle.qmv(w["fmt"], W, w["rows"], w["cols"], x)
    within(y, ref, bound)


def test_cfg1_fused_qkv_equals_the_three_projections():
    w = synth.workload_cfg1()
    fmt, rows, cols = w["fmt"], w["rows"], w["cols"]
    W = synth.gen_blocks(fmt, rows, cols, w["seed"], 0)
    x = synth.gen_x(1, cols, w["seed"], 1)
    y = run_qmv(fmt, W, rows, cols, x)
    ref, bound = oracle.qmv(fmt, W, rows, cols, x)
    within(y, ref, bound)
    rb = synth.matrix_bytes(fmt, 1, cols)
    parts = [run_qmv(fmt, W[a * rb:b * rb], b - a, cols, x) for _, a, b in w["segments"]]
    within(np.concatenate(parts, axis=1), ref, bound)


@pytest.mark.parametrize("n_tok", [1, 4])
def test_cfg2_q6_k_vocab_projection_sampled_rows(n_tok):
    w = synth.workload_cfg2(n_tok)
    fmt, rows, cols = w["fmt"], w["rows"], w["cols"]
    W = synth.gen_blocks(fmt, rows, cols, w["seed"], 0)
    x = synth.gen_x(n_tok, cols, w["seed"], 1)
    y = run_qmv(fmt, W, rows, cols, x)
    idx = np.unique(np.concatenate([np.arange(64), np.arange(rows - 64, rows),
                                    np.random.default_rng(n_tok).integers(0, rows, 4000)]))
    ref, bound = oracle.qmv_rows(fmt, W, rows, cols, idx, x)
    within(y[:, idx], ref, bound)


@pytest.mark.parametrize("n_tok", [1, 2, 4, 8])
def test_cfg4_q8_0_layer_matvecs(n_tok):
    # layer 0 of the 16-layer Q8_0 stack: every row; the bench times the same calls
    for m, (name, rows, cols) in enumerate(synth.workload_cfg4_layer()):
        W = synth.gen_blocks(Q8_0, rows, cols, synth.CFG4_SEED, m)
        x = synth.gen_x(n_tok, cols, synth.CFG4_SEED, 1000 + m)
        y = run_qmv(Q8_0, W, rows, cols, x)
        if rows * cols <= 3072 * 2048 or n_tok == 1:
            ref, bound = oracle.qmv(Q8_0, W, rows, cols, x, nthreads=8)
            within(y, ref, bound)
        else:
            idx = np.random.default_rng(m).integers(0, rows, 1024)
            ref, bound = oracle.qmv_rows(Q8_0, W, rows, cols, idx, x)
            within(y[:, idx], ref, bound)


# --------------------------------------------------------------------- MoE --

def _router_case(seed):
    logits, bias = synth.gen_router(32, seed, 5)
    ids, g, biased = oracle.route(logits, bias, 4)
    srt = np.sort(biased.astype(np.float64))[::-1]
    assert srt[3] - srt[4] > 1e-5, "ambiguous top-4 cut for this seed"
    return logits, bias, ids, g


@pytest.mark.parametrize("seed", [3, 4, 5, 6, 7, 8, 9, 10])
def test_router_matches_oracle(seed):
    logits, bias, ids, g = _router_case(seed)
    ids_d = torch.empty(4, dtype=torch.int32, device="cuda")
    g_d = torch.empty(4, device="cuda")
    q.moe_route(dev(logits), dev(bias), 32, 4, ids_d, g_d)
    torch.cuda.synchronize()
    assert ids_d.cpu().tolist() == ids.tolist()
    assert np.allclose(g_d.cpu().numpy(), g, rtol=1e-6, atol=0)


def test_router_other_sizes_and_ties():
    logits = np.zeros(40, np.float32)
    bias = np.zeros(40, np.float32)
    bias[[3, 17, 39]] = 1.0
    ids_d = torch.empty(5, dtype=torch.int32, device="cuda")
    g_d = torch.empty(5, device="cuda")
    q.moe_route(dev(logits), dev(bias), 40, 5, ids_d, g_d)
    torch.cuda.synchronize()
    ids, g, _ = oracle.route(logits, bias, 5)
    assert ids_d.cpu().tolist() == ids.tolist() == [3, 17, 39, 0, 1]
    assert np.allclose(g_d.cpu().numpy(), 0.2, rtol=1e-6)


def _moe_weights(n_expert, hidden, inter, seed):
    gus = synth.matrix_bytes(Q4_K, inter, hidden)
    ds = synth.matrix_bytes(Q4_K, hidden, inter)
    gate = synth.gen_blocks(Q4_K, inter * n_expert, hidden, seed, 1)
    up = synth.gen_blocks(Q4_K, inter * n_expert, hidden, seed, 2)
    down = synth.gen_blocks(Q4_K, hidden * n_expert, inter, seed, 3)
    x = synth.gen_x(1, hidden, seed, 4)[0]
    return gate, up, down, gus, ds, x


def test_moe_qmv_separate_and_weighted():
    n_expert, rows, cols = 8, 300, 1792
    mb = synth.matrix_bytes(Q4_K, rows, cols)
    E = synth.gen_blocks(Q4_K, rows * n_expert, cols, 40, 1)
    ids = np.array([5, 0, 7, 2], np.int32)
    xs = synth.gen_x(4, cols, 40, 2)
    gw = np.array([0.1, 0.2, 0.3, 0.4], np.float32)
    # separate: y[k] = W_{ids[k]} x_k
    y = torch.empty((4, rows), device="cuda")
    q.moe_qmv(Q4_K, dev(E), mb, n_expert, dev(ids), 4, rows, cols, dev(xs), cols, None, y)
    yw = torch.empty(rows, device="cuda")
    q.moe_qmv(Q4_K, dev(E), mb, n_expert, dev(ids), 4, rows, cols, dev(xs), cols, dev(gw), yw)
    # shared x (x_stride 0), weighted
    ys = torch.empty(rows, device="cuda")
    q.moe_qmv(Q4_K, dev(E), mb, n_expert, dev(ids[:3]), 3, rows, cols, dev(xs[0]), 0, dev(gw[:3]), ys)
    torch.cuda.synchronize()
    refs, bounds = [], []
    for k, e in enumerate(ids):
        r, b = oracle.qmv(Q4_K, E[e * mb:(e + 1) * mb], rows, cols, xs[k])
        refs.append(r[0]); bounds.append(b[0])
    within(y.cpu().numpy(), np.array(refs), np.array(bounds))
    wsum = sum(float(gw[k]) * refs[k] for k in range(4))
    wb = sum(abs(float(gw[k])) * bounds[k] for k in range(4))
    within(yw.cpu().numpy(), wsum, wb)
    r3 = [oracle.qmv(Q4_K, E[e * mb:(e + 1) * mb], rows, cols, xs[0]) for e in ids[:3]]
    within(ys.cpu().numpy(), sum(float(gw[k]) * r3[k][0][0] for k in range(3)),
           sum(abs(float(gw[k])) * r3[k][1][0] for k in range(3)))


def test_moe_bad_expert_id_is_dropped_and_reported():
    n_expert, rows, cols = 4, 64, 256
    mb = synth.matrix_bytes(Q4_K, rows, cols)
    E = synth.gen_blocks(Q4_K, rows * n_expert, cols, 41, 1)
    x = synth.gen_x(1, cols, 41, 2)
    y = torch.full((2, rows), 5.0, device="cuda")
    q.moe_qmv(Q4_K, dev(E), mb, n_expert, dev(np.array([1, 9], np.int32)), 2, rows, cols,
              dev(x), 0, None, y)
    err = q.qmv_check()
    assert err & q.DEVERR_EXPERT_ID
    assert q.qmv_check() == 0                      # cleared by the read
    ref, bound = oracle.qmv(Q4_K, E[mb:2 * mb], rows, cols, x)
    yh = y.cpu().numpy()
    within(yh[:1], ref, bound)
    assert np.array_equal(yh[1], np.zeros(rows, np.float32))


@pytest.mark.parametrize("fmt,rows,cols,n_tok,kernel", [(Q8_0, 512, 2048, 1, q.KERNEL_STREAM),
                                                     (Q8_0, 512, 2048, 2, q.KERNEL_STREAM),
                                                     (Q6_K, 300, 8192, 4, q.KERNEL_WARP_RING),
                                                     (Q8_0, 512, 2048, 8, q.KERNEL_TENSOR_CORE)])
def test_stage_wait_timeout_is_reported_and_the_gpu_stays_usable(fmt, rows, cols, n_tok, kernel):
    # the test hook makes every tile expect 16 bytes more than are copied
    # (the streaming kernel at one and two tokens, the warp-ring kernel, the
    # tensor-core kernel): each stage wait runs out (about a second), the
    # kernel records the timeout and finishes, and the context stays usable
    W = synth.gen_blocks(fmt, rows, cols, 45, 0)
    x = synth.gen_x(n_tok, cols, 45, 1)
    y = torch.empty((n_tok, rows), device="cuda")
    q.lib().qmv_debug_short_copies(16)
    try:
        if n_tok == 1:
            q.qmv_f32(fmt, dev(W), rows, cols, dev(x), y)
        else:
            q.qmv_batched(fmt, dev(W), rows, cols, dev(x), y, n_tok)
        assert q.qmv_debug_last_kernel() == kernel
        err = q.qmv_check()
    finally:
        q.lib().qmv_debug_short_copies(0)
    assert err & q.DEVERR_TIMEOUT
    assert q.qmv_check() == 0                      # cleared by the read
    ref, bound = oracle.qmv(fmt, W, rows, cols, x)
    within(run_qmv(fmt, W, rows, cols, x), ref, bound)


def _check_moe_ffn(n_expert, hidden, inter, seed, ids, g32):
    gate, up, down, gus, ds, x = _moe_weights(n_expert, hidden, inter, seed)
    n_sel = len(ids)
    h = torch.empty((n_sel, inter), device="cuda")
    y = torch.empty(hidden, device="cuda")
    q.moe_ffn(Q4_K, dev(gate), dev(up), gus, Q4_K, dev(down), ds, n_expert,
              dev(np.asarray(ids, np.int32)), dev(g32), n_sel, hidden, inter, dev(x), h, y)
    torch.cuda.synchronize()
    hg, yg = h.cpu().numpy(), y.cpu().numpy()
    g64 = g32.astype(np.float64)
    full = oracle.moe_ffn(Q4_K, gate, up, gus, Q4_K, down, ds, n_expert, ids, g64, hidden, inter, x)
    # (i) h_k = silu(u_k) v_k, with u_k and v_k each held to the single-matvec rule
    y_ref2 = np.zeros(hidden)
    b2 = np.zeros(hidden)
    prop = np.zeros(hidden)
    for k, e in enumerate(ids):
        _, bu = oracle.qmv(Q4_K, gate[e * gus:(e + 1) * gus], inter, hidden, x)
        _, bv = oracle.qmv(Q4_K, up[e * gus:(e + 1) * gus], inter, hidden, x)
        du, dv = REL * bu[0] + ABS, REL * bv[0] + ABS
        u, v = full["u"][k], full["v"][k]
        su = u / (1 + np.exp(-u))
        dh = 1.1 * du * np.abs(v) + np.abs(su) * dv + 1.1 * du * dv + 1e-6 * np.abs(full["h"][k])
        err = np.abs(hg[k] - full["h"][k])
        assert (err <= dh + ABS).all(), f"h_{k}: worst {(err / (dh + ABS)).max():.3g}"
        # (ii) the down stage fed the GPU's own h_k
        Dk = down[e * ds:(e + 1) * ds]
        r, b = oracle.qmv(Q4_K, Dk, hidden, inter, hg[k])
        y_ref2 += g64[k] * r[0]
        b2 += abs(g64[k]) * b[0]
        prop += abs(g64[k]) * (np.abs(oracle.dequant(Q4_K, Dk, hidden, inter).astype(np.float64)) @ dh)
    within(yg, y_ref2, b2)
    # (iii) end to end against the all-f64 oracle, the bound widened by the h error
    err = np.abs(yg - full["y"])
    assert (err <= REL * b2 + ABS + prop).all()


def test_moe_ffn_cfg3_routed_on_device():
    w = synth.workload_cfg3()
    n_expert, hidden, inter, seed = w["n_expert"], w["hidden"], w["inter"], w["seed"]
    logits, bias, ids, g = _router_case(seed)
    # route on the device, then the FFN step from the device ids / weights
    gate, up, down, gus, ds, x = _moe_weights(n_expert, hidden, inter, seed)
    ids_d = torch.empty(4, dtype=torch.int32, device="cuda")
    g_d = torch.empty(4, device="cuda")
    q.moe_route(dev(logits), dev(bias), n_expert, 4, ids_d, g_d)
    h = torch.empty((4, inter), device="cuda")
    y = torch.empty(hidden, device="cuda")
    q.moe_ffn(Q4_K, dev(gate), dev(up), gus, Q4_K, dev(down), ds, n_expert, ids_d, g_d, 4,
              hidden, inter, dev(x), h, y)
    torch.cuda.synchronize()
    assert ids_d.cpu().tolist() == ids.tolist()
    y_dev = y.cpu().numpy()
    # the same step with the oracle's ids and the device's weights, checked in full
    _check_moe_ffn(n_expert, hidden, inter, seed, ids.tolist(), g_d.cpu().numpy())
    h2 = torch.empty((4, inter), device="cuda")
    y2 = torch.empty(hidden, device="cuda")
    q.moe_ffn(Q4_K, dev(gate), dev(up), gus, Q4_K, dev(down), ds, n_expert, dev(ids), g_d, 4,
              hidden, inter, dev(x), h2, y2)
    torch.cuda.synchronize()
    assert np.array_equal(y2.cpu().numpy().view(np.uint32), y_dev.view(np.uint32))


@pytest.mark.parametrize("ids", [[2], [0, 3], [1, 2, 3], [4, 0, 6, 1, 5, 7, 3, 2]])
def test_moe_ffn_other_expert_counts(ids):
    g = np.random.default_rng(len(ids)).uniform(0.1, 1.0, len(ids)).astype(np.float32)
    _check_moe_ffn(8, 512, 768, 50 + len(ids), ids, g)


@pytest.mark.parametrize("fmt,hidden,inter,kernel", [(Q4_K, 2048, 1792, q.KERNEL_STREAM),
                                                     (Q8_0, 1024, 512, q.KERNEL_STREAM),
                                                     (Q8_0, 4096, 1024, q.KERNEL_STREAM),
                                                     (Q4_K, 512, 2304, q.KERNEL_GENERAL)])
def test_moe_ffn_formats_and_a_bad_expert_id(fmt, hidden, inter, kernel):
    # Q8_0 experts, rows of more than one K-segment (hidden 4096), expert rows
    # longer than one K-segment (inter 2304: the general kernel), and an expert
    # id out of range: that expert contributes nothing (h row zero) and is
    # reported
    n_expert, ids, g32 = 6, [4, 1, 9, 3], np.array([0.4, 0.3, 0.2, 0.1], np.float32)
    gus, ds = synth.matrix_bytes(fmt, inter, hidden), synth.matrix_bytes(fmt, hidden, inter)
    gate = synth.gen_blocks(fmt, inter * n_expert, hidden, 61, 1)
    up = synth.gen_blocks(fmt, inter * n_expert, hidden, 61, 2)
    down = synth.gen_blocks(fmt, hidden * n_expert, inter, 61, 3)
    x = synth.gen_x(1, hidden, 61, 4)[0]
    h = torch.full((4, inter), float("nan"), device="cuda")
    y = torch.full((hidden,), float("nan"), device="cuda")
    q.moe_ffn(fmt, dev(gate), dev(up), gus, fmt, dev(down), ds, n_expert, dev(np.array(ids, np.int32)),
              dev(g32), 4, hidden, inter, dev(x), h, y)
    assert q.qmv_debug_last_kernel() == kernel
    err = q.qmv_check()
    assert err & q.DEVERR_EXPERT_ID
    hh, yy = h.cpu().numpy(), y.cpu().numpy()
    assert np.array_equal(hh[2], np.zeros(inter, np.float32))
    good = [0, 1, 3]
    ref = oracle.moe_ffn(fmt, gate, up, gus, fmt, down, ds, n_expert, np.array([ids[k] for k in good]),
                         g32[good].astype(np.float64), hidden, inter, x)
    # h of the valid experts: the composite rule (i) of _check_moe_ffn
    for j, k in enumerate(good):
        e = ids[k]
        _, bu = oracle.qmv(fmt, gate[e * gus:(e + 1) * gus], inter, hidden, x)
        _, bv = oracle.qmv(fmt, up[e * gus:(e + 1) * gus], inter, hidden, x)
        du, dv = REL * bu[0] + ABS, REL * bv[0] + ABS
        u, v = ref["u"][j], ref["v"][j]
        su = u / (1 + np.exp(-u))
        dh = 1.1 * du * np.abs(v) + np.abs(su) * dv + 1.1 * du * dv + 1e-6 * np.abs(ref["h"][j])
        assert (np.abs(hh[k] - ref["h"][j]) <= dh + ABS).all(), k
    # y from the GPU's own h: the weighted down sum over the valid experts
    yref = np.zeros(hidden)
    bnd = np.zeros(hidden)
    for k in good:
        r, b = oracle.qmv(fmt, down[ids[k] * ds:(ids[k] + 1) * ds], hidden, inter, hh[k][None, :])
        yref += float(g32[k]) * r[0]
        bnd += abs(float(g32[k])) * b[0]
    within(yy[None, :], yref[None, :], bnd[None, :])
    assert np.isfinite(ref["y"]).all()


@pytest.mark.parametrize("fmt,n_expert,hidden,inter,top_k,seed", [(Q4_K, 32, 2048, 1792, 4, 3),
                                                                  (Q8_0, 16, 1024, 512, 3, 71),
                                                                  (Q4_K, 8, 4096, 768, 6, 72),
                                                                  (Q4_K, 8, 512, 2304, 4, 73)])
def test_moe_ffn_routed_matches_route_then_ffn(fmt, n_expert, hidden, inter, top_k, seed):
    # the one-launch step (router in every CTA, grid barrier between the two
    # products) against moe_route followed by moe_ffn: the same ids and
    # weights, and bit-identical h and y (the same decode and reduction order);
    # expert rows of 2304 columns take the two-launch path instead
    gus, ds = synth.matrix_bytes(fmt, inter, hidden), synth.matrix_bytes(fmt, hidden, inter)
    gate = dev(synth.gen_blocks(fmt, inter * n_expert, hidden, seed, 1))
    up = dev(synth.gen_blocks(fmt, inter * n_expert, hidden, seed, 2))
    down = dev(synth.gen_blocks(fmt, hidden * n_expert, inter, seed, 3))
    ws = torch.zeros(q.MOE_WS_BYTES // 8, dtype=torch.int64, device="cuda")
    for call in range(2):
        logits, bias = synth.gen_router(n_expert, seed + call, 5)
        lg, bs = dev(logits), dev(bias)
        x = dev(synth.gen_x(1, hidden, seed + call, 4)[0])
        ids_a = torch.empty(top_k, dtype=torch.int32, device="cuda")
        g_a = torch.empty(top_k, device="cuda")
        h_a = torch.empty((top_k, inter), device="cuda")
        y_a = torch.empty(hidden, device="cuda")
        q.moe_route(lg, bs, n_expert, top_k, ids_a, g_a)
        q.moe_ffn(fmt, gate, up, gus, fmt, down, ds, n_expert, ids_a, g_a, top_k, hidden, inter, x, h_a, y_a)
        ids_b = torch.full((top_k,), -9, dtype=torch.int32, device="cuda")
        g_b = torch.full((top_k,), float("nan"), device="cuda")
        h_b = torch.full((top_k, inter), float("nan"), device="cuda")
        y_b = torch.full((hidden,), float("nan"), device="cuda")
        q.moe_ffn_routed(lg, bs, n_expert, top_k, fmt, gate, up, gus, fmt, down, ds, hidden, inter, x,
                         ids_b, g_b, h_b, y_b, ws)
        assert q.qmv_debug_last_kernel() == (q.KERNEL_STREAM if inter <= 2048 else q.KERNEL_GENERAL)
        torch.cuda.synchronize()
        assert ids_b.cpu().tolist() == ids_a.cpu().tolist()
        assert np.array_equal(g_b.cpu().numpy().view(np.uint32), g_a.cpu().numpy().view(np.uint32))
        assert np.array_equal(h_b.cpu().numpy().view(np.uint32), h_a.cpu().numpy().view(np.uint32))
        assert np.array_equal(y_b.cpu().numpy().view(np.uint32), y_a.cpu().numpy().view(np.uint32))
        assert int(ws.abs().sum().cpu()) == 0
    assert q.qmv_check() == 0
