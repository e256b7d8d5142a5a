"""Pins of the oracle to things other than itself (CPU only, no GPU).

Each check is chosen so that a plausible slip in the oracle -- a field read
from the wrong byte or bit, a dropped term (the min, the -32 offset), a wrong
sign, a swapped token/column index, a wrong tie rule -- fails at least one of
them.  Sources: per-slot round trips through the test-side encoder, a second
bit-string decoder, numpy's float16 cast, hand-worked blocks, closed forms,
exact rational brute force, the page-printed constants, and brute-force subset
search for the router.
"""
from __future__ import annotations

import itertools
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle
from blockpack import (decode2, f16_bits, fields_q4_k, fields_q6_k, fields_q8_0,
                       pack_q4_k, pack_q6_k, pack_q8_0)
from quantized_decode_superblocks_b200 import synth

Q8_0, Q4_K, Q6_K = oracle.Q8_0, oracle.Q4_K, oracle.Q6_K
ONE = f16_bits(1.0)
ZERO = f16_bits(0.0)


def golden_constants():
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "page_constants.txt")
    out = {}
    for line in open(path, encoding="utf-8"):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        name, value = line.split()[:2]
        out[name] = int(value)
    return out


# ------------------------------------------------------------- fp16 decode --

def test_fp16_decode_all_patterns_match_numpy():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float32)
    got = np.array([oracle.half_to_float(int(b)) for b in bits], dtype=np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


# ------------------------------------------------------- sizes (the pages) --

def test_block_sizes_against_page_constants():
    c = golden_constants()
    assert oracle.block_weights(Q4_K) == c["q4k_weights_per_superblock"]
    assert oracle.block_bytes(Q4_K) == c["q4k_bytes_per_superblock"]
    # 4.5 bits per weight follows from 144 B / 256 weights
    assert oracle.block_bytes(Q4_K) * 8 / oracle.block_weights(Q4_K) == 4.5
    assert (oracle.block_weights(Q8_0), oracle.block_bytes(Q8_0)) == (32, 34)
    assert (oracle.block_weights(Q6_K), oracle.block_bytes(Q6_K)) == (256, 210)
    assert oracle.block_weights(7) == 0 and oracle.block_bytes(7) == 0


def test_fusion_call_count_matches_page():
    # unfused layer: q, k, v, o, gate, up, down; fused: qkv, o, gate_up, down
    c = golden_constants()
    fused = synth.workload_cfg4_layer()
    assert len(fused) == 4
    assert round(100 * (1 - len(fused) / 7)) == c["fused_matvec_call_cut_percent"]
    qkv = synth.workload_cfg1()
    head_dim = 64
    assert qkv["rows"] == (c["query_heads"] + 2 * c["kv_heads"]) * head_dim
    assert qkv["cols"] == c["hidden"]


# --------------------------------------------------- per-slot round trips --

def _dequant_blocks(fmt, blocks):
    """Dequantize a list of blocks (one block per row) in a single oracle call."""
    W = np.concatenate(blocks)
    bw = oracle.block_weights(fmt)
    return oracle.dequant(fmt, W, len(blocks), bw)


def test_q8_0_every_slot_every_value():
    blocks, expect = [], []
    for i in range(32):
        for v in range(-128, 128):
            q = [0] * 32
            q[i] = v
            blocks.append(pack_q8_0(ONE, q))
            e = np.zeros(32, np.float32)
            e[i] = v
            expect.append(e)
    got = _dequant_blocks(Q8_0, blocks)
    assert np.array_equal(got, np.array(expect))


def test_q8_0_scale_is_applied():
    # d = 0.5 halves every weight; d = -2 flips the sign
    q = list(range(-16, 16))
    for d, mul in ((0.5, 0.5), (-2.0, -2.0)):
        got = oracle.dequant_block(Q8_0, pack_q8_0(f16_bits(d), q))
        assert np.array_equal(got, np.array(q, np.float32) * np.float32(mul))


def test_q4_k_every_scale_and_min_slot_every_value():
    blocks, expect = [], []
    for j in range(8):
        for v in range(64):
            sc = [0] * 8
            sc[j] = v
            blocks.append(pack_q4_k(ONE, ZERO, sc, [0] * 8, [1] * 256))
            e = np.zeros(256, np.float32)
            e[32 * j:32 * j + 32] = v
            expect.append(e)
            m = [0] * 8
            m[j] = v
            blocks.append(pack_q4_k(ZERO, ONE, [0] * 8, m, [1] * 256))
            e = np.zeros(256, np.float32)
            e[32 * j:32 * j + 32] = -v
            expect.append(e)
    got = _dequant_blocks(Q4_K, blocks)
    assert np.array_equal(got, np.array(expect))


def test_q4_k_every_nibble_position_every_value():
    blocks, expect = [], []
    for i in range(256):
        for v in range(16):
            q = [0] * 256
            q[i] = v
            blocks.append(pack_q4_k(ONE, ZERO, [1] * 8, [0] * 8, q))
            e = np.zeros(256, np.float32)
            e[i] = v
            expect.append(e)
    got = _dequant_blocks(Q4_K, blocks)
    assert np.array_equal(got, np.array(expect))


def test_q6_k_every_position_every_quant():
    blocks, expect = [], []
    for i in range(256):
        for v in range(64):
            q = [32] * 256
            q[i] = v
            blocks.append(pack_q6_k(ONE, [1] * 16, q))
            e = np.zeros(256, np.float32)
            e[i] = v - 32
            expect.append(e)
    got = _dequant_blocks(Q6_K, blocks)
    assert np.array_equal(got, np.array(expect))


def test_q6_k_every_scale_slot_every_value():
    blocks, expect = [], []
    for k in range(16):
        for v in range(-128, 128):
            s = [0] * 16
            s[k] = v
            blocks.append(pack_q6_k(ONE, s, [33] * 256))
            e = np.zeros(256, np.float32)
            e[16 * k:16 * k + 16] = v
            expect.append(e)
    got = _dequant_blocks(Q6_K, blocks)
    assert np.array_equal(got, np.array(expect))


# ------------------------------------------------------- second decoder --

@pytest.mark.parametrize("fmt", [Q8_0, Q4_K, Q6_K])
def test_second_decoder_agrees_bit_for_bit(fmt):
    bw, bb = oracle.block_weights(fmt), oracle.block_bytes(fmt)
    W = synth.gen_blocks(fmt, 40, bw * 3, seed=11, tensor_id=fmt)
    got = oracle.dequant(fmt, W, 40, bw * 3).reshape(-1, bw)
    for k in range(W.size // bb):
        ref = decode2(fmt, W[k * bb:(k + 1) * bb])
        assert np.array_equal(got[k].view(np.uint32), ref.view(np.uint32)), k


def test_synth_fields_follow_their_distributions():
    n = 4000
    f8 = [fields_q8_0(b) for b in synth.gen_blocks(Q8_0, n, 32, 5, 0).reshape(n, 34)]
    ds = np.array([f["d"] for f in f8])
    qs = np.array([f["q"] for f in f8])
    assert ds.min() >= 1e-3 - 1e-6 and ds.max() <= 2e-2 + 1e-5
    assert qs.min() == -127 and qs.max() == 127
    f4 = [fields_q4_k(b) for b in synth.gen_blocks(Q4_K, 500, 256, 5, 1).reshape(500, 144)]
    sc = np.array([f["sc"] + f["m"] for f in f4])
    assert sc.min() == 0 and sc.max() == 63 and abs(sc.mean() - 31.5) < 1.0
    assert min(f["dmin"] for f in f4) >= 1e-3 - 1e-6 and max(f["d"] for f in f4) <= 1e-2 + 1e-5
    f6 = [fields_q6_k(b) for b in synth.gen_blocks(Q6_K, 500, 256, 5, 2).reshape(500, 210)]
    s6 = np.array([f["scales"] for f in f6])
    q6 = np.array([f["q"] for f in f6])
    assert s6.min() == -64 and s6.max() == 63
    assert q6.min() == 0 and q6.max() == 63 and abs(q6.mean() - 31.5) < 0.5


# ------------------------------------------------------ hand-worked blocks --

def test_hand_worked_q4_k_block():
    # d = 1, dmin = 0.5, sc_j = j + 1, m_j = 2j, q_i = i mod 16
    # => w_i = (j+1)(i mod 16) - j with j = i // 32, worked by hand:
    blk = pack_q4_k(ONE, f16_bits(0.5), [j + 1 for j in range(8)], [2 * j for j in range(8)],
                    [i % 16 for i in range(256)])
    w = oracle.dequant_block(Q4_K, blk)
    for i, val in {0: 0, 17: 1, 35: 5, 100: 13, 191: 85, 224: -7, 255: 113}.items():
        assert w[i] == val, i


def test_hand_worked_q6_k_block():
    # d = 0.25, scales[k] = -64 + k, q_i = i mod 64
    # => w_i = 0.25 * (-64 + i // 16) * (i mod 64 - 32), worked by hand:
    blk = pack_q6_k(f16_bits(0.25), [-64 + k for k in range(16)], [i % 64 for i in range(256)])
    w = oracle.dequant_block(Q6_K, blk)
    for i, val in {0: 512.0, 31: 15.75, 32: 0.0, 100: -58.0, 129: 434.0, 255: -379.75}.items():
        assert w[i] == val, i


def test_hand_worked_q8_0_block():
    # d = 0.5, q_i = i - 16  => w_0 = -8, w_16 = 0, w_31 = 7.5
    w = oracle.dequant_block(Q8_0, pack_q8_0(f16_bits(0.5), [i - 16 for i in range(32)]))
    assert (w[0], w[16], w[31]) == (-8.0, 0.0, 7.5)


def test_q4_k_single_rounding_of_the_difference():
    # d*sc*q and dmin*m are exact; only the difference rounds, to nearest even.
    # d = 1, sc = 2, q = 1 gives 2; dmin = 2^-24 (smallest fp16 subnormal).
    # Just below 2 the f32 spacing is 2^-23, so
    #   m = 1: 2 - 2^-24   is a tie between 2 - 2^-23 (odd) and 2 (even)  -> 2
    #   m = 2: 2 - 2^-23   is exact
    #   m = 3: 2 - 3*2^-24 is a tie between 2 - 2^-23 (odd) and 2 - 2^-22 (even)
    blk = pack_q4_k(ONE, f16_bits(2.0 ** -24), [2] * 8, [1, 2, 3, 0, 0, 0, 0, 0], [1] * 256)
    w = oracle.dequant_block(Q4_K, blk)
    assert w[0] == 2.0
    assert w[32] == np.float32(2 - 2.0 ** -23)
    assert w[64] == np.float32(2 - 2.0 ** -22)
    assert w[96] == 2.0


# ------------------------------------------------------------ closed forms --

def _sum_x(x):
    return float(np.sum(x.astype(np.float64)))


@pytest.mark.parametrize("Q,S,M", [(0, 5, 7), (15, 63, 0), (9, 17, 63), (7, 0, 11)])
def test_q4_k_constant_fields_closed_form(Q, S, M):
    d, dmin = 0.0078125, 0.00390625        # exact in fp16
    rows, cols = 3, 512
    blk = pack_q4_k(f16_bits(d), f16_bits(dmin), [S] * 8, [M] * 8, [Q] * 256)
    W = np.tile(blk, rows * cols // 256)
    x = synth.gen_x(2, cols, 7, 0)
    y, _ = oracle.qmv(Q4_K, W, rows, cols, x)
    for t in range(2):
        ref = (d * S * Q - dmin * M) * _sum_x(x[t])
        assert np.allclose(y[t], ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("Q,s", [(0, 1), (63, -64), (32, 17), (45, -3)])
def test_q6_k_constant_fields_closed_form(Q, s):
    d = 0.001953125
    rows, cols = 2, 768
    blk = pack_q6_k(f16_bits(d), [s] * 16, [Q] * 256)
    W = np.tile(blk, rows * cols // 256)
    x = synth.gen_x(1, cols, 8, 0)
    y, _ = oracle.qmv(Q6_K, W, rows, cols, x)
    assert np.allclose(y, d * s * (Q - 32) * _sum_x(x[0]), rtol=1e-12, atol=1e-12)


def test_q8_0_unit_scale_integer_dot_is_exact():
    g = np.random.default_rng(3)
    rows, cols = 5, 96
    q = g.integers(-127, 128, size=(rows, cols))
    W = np.concatenate([pack_q8_0(ONE, q[r, 32 * b:32 * b + 32]) for r in range(rows) for b in range(3)])
    x = g.integers(-8, 9, size=(1, cols)).astype(np.float32)
    y, _ = oracle.qmv(Q8_0, W, rows, cols, x)
    exact = [sum(int(q[r, i]) * int(x[0, i]) for i in range(cols)) for r in range(rows)]
    assert y[0].tolist() == [float(e) for e in exact]


def test_zero_scale_gives_zero_and_zero_sc_leaves_the_min_term():
    x = synth.gen_x(1, 256, 9, 0)
    blk = pack_q8_0(ZERO, list(range(-16, 16)))
    y, b = oracle.qmv(Q8_0, np.tile(blk, 8), 1, 256, x)
    assert y[0, 0] == 0.0 and b[0, 0] == 0.0
    blk = pack_q4_k(f16_bits(0.5), f16_bits(0.25), [0] * 8, [6] * 8, list(range(16)) * 16)
    y, _ = oracle.qmv(Q4_K, blk, 1, 256, x)
    assert np.isclose(y[0, 0], -0.25 * 6 * _sum_x(x[0]), rtol=1e-12, atol=1e-12)


# --------------------------------------------------- exact brute force ----

def _exact_rows(fmt, blocks_fields, cols, xs):
    """Exact rational y and bound from FIELDS (not from the oracle's decode)."""
    ys, bs = [], []
    for t in range(xs.shape[0]):
        xf = [Fraction(float(v)) for v in xs[t]]
        yr, br = [], []
        for fields in blocks_fields:
            w = []
            for f in fields:
                if fmt == Q8_0:
                    w += [Fraction(f["d"]) * q for q in f["q"]]
                elif fmt == Q4_K:
                    for i in range(256):
                        exact = (Fraction(f["d"]) * f["sc"][i // 32] * f["q"][i]
                                 - Fraction(f["dmin"]) * f["m"][i // 32])
                        assert Fraction(float(exact)) == exact   # f64 holds it exactly
                        w.append(Fraction(float(np.float32(float(exact)))))
                else:
                    w += [Fraction(f["d"]) * f["scales"][i // 16] * (f["q"][i] - 32) for i in range(256)]
            yr.append(sum(wi * xi for wi, xi in zip(w, xf)))
            br.append(sum(abs(wi * xi) for wi, xi in zip(w, xf)))
        ys.append(yr)
        bs.append(br)
    return ys, bs


@pytest.mark.parametrize("fmt,rows", [(Q8_0, 1), (Q8_0, 3), (Q4_K, 1), (Q4_K, 3), (Q6_K, 1), (Q6_K, 3)])
def test_brute_force_exact_rational(fmt, rows):
    bw, bb = oracle.block_weights(fmt), oracle.block_bytes(fmt)
    nb = 2 if fmt == Q8_0 else 1
    cols = bw * nb
    g = np.random.default_rng(100 + 10 * fmt + rows)
    blocks, fields = [], []
    for r in range(rows):
        row_fields = []
        for b in range(nb):
            if fmt == Q8_0:
                d = float(np.float16(g.uniform(1e-3, 2e-2)))
                q = g.integers(-127, 128, size=32)
                blk = pack_q8_0(f16_bits(d), q)
            elif fmt == Q4_K:
                blk = pack_q4_k(f16_bits(g.uniform(1e-3, 1e-2)), f16_bits(g.uniform(1e-3, 1e-2)),
                                g.integers(0, 64, 8), g.integers(0, 64, 8), g.integers(0, 16, 256))
            else:
                blk = pack_q6_k(f16_bits(g.uniform(1e-4, 2e-3)), g.integers(-64, 64, 16),
                                g.integers(0, 64, 256))
            blocks.append(blk)
            row_fields.append({Q8_0: fields_q8_0, Q4_K: fields_q4_k, Q6_K: fields_q6_k}[fmt](blk))
        fields.append(row_fields)
    W = np.concatenate(blocks)
    x = g.standard_normal((3, cols)).astype(np.float32)   # 3 distinct tokens
    y, b = oracle.qmv(fmt, W, rows, cols, x)
    ys, bs = _exact_rows(fmt, fields, cols, x)
    gamma = cols * 2.0 ** -53 / (1 - cols * 2.0 ** -53)
    for t in range(3):
        for r in range(rows):
            ex, mag = ys[t][r], bs[t][r]
            assert abs(Fraction(y[t, r]) - ex) <= Fraction(gamma) * mag + Fraction(1, 10 ** 300)
            assert abs(Fraction(b[t, r]) - mag) <= Fraction(gamma) * mag + Fraction(1, 10 ** 300)
    # sampled-row entry point agrees with the full one
    yr, br = oracle.qmv_rows(fmt, W, rows, cols, list(range(rows))[::-1], x)
    assert np.array_equal(yr, y[:, ::-1]) and np.array_equal(br, b[:, ::-1])


def test_multi_token_is_per_token():
    fmt, rows, cols = Q4_K, 6, 512
    W = synth.gen_blocks(fmt, rows, cols, 12, 0)
    x = synth.gen_x(5, cols, 12, 1)
    y, b = oracle.qmv(fmt, W, rows, cols, x)
    for t in range(5):
        y1, b1 = oracle.qmv(fmt, W, rows, cols, x[t])
        assert np.array_equal(y1[0], y[t]) and np.array_equal(b1[0], b[t])
    # the row-parallel build does the same arithmetic
    y8, b8 = oracle.qmv(fmt, W, rows, cols, x, nthreads=4)
    assert np.array_equal(y8, y) and np.array_equal(b8, b)


def test_bad_arguments_are_rejected():
    W = np.zeros(34, np.uint8)
    with pytest.raises(ValueError):
        oracle.qmv(Q8_0, W, 1, 33, np.zeros(33, np.float32))
    with pytest.raises(ValueError):
        oracle.qmv(9, W, 1, 32, np.zeros(32, np.float32))


# ------------------------------------------------------------------ router --

def _sigmoid64(v):
    return 1.0 / (1.0 + math.exp(-float(v)))


@pytest.mark.parametrize("seed", range(6))
def test_router_matches_subset_brute_force(seed):
    c = golden_constants()
    n, k = c["moe_experts"], c["moe_top_k"]
    logits, bias = synth.gen_router(n, 50 + seed, 0)
    ids, g, biased = oracle.route(logits, bias, k)
    b64 = np.array([_sigmoid64(l) + float(bb) for l, bb in zip(logits, bias)])
    order = np.sort(b64)[::-1]
    assert order[k - 1] - order[k] > 1e-6            # no near-tie at the cut
    best = max(itertools.combinations(range(n), k), key=lambda s: sum(b64[list(s)]))
    assert set(ids.tolist()) == set(best)
    assert list(ids) == sorted(ids.tolist(), key=lambda e: -b64[e])   # descending order
    s = np.array([_sigmoid64(logits[e]) for e in ids])
    assert np.allclose(g, s / s.sum(), rtol=1e-15)
    assert abs(g.sum() - 1.0) < 1e-15
    assert np.allclose(biased, b64, atol=1e-6)


def test_router_bias_selects_but_does_not_weight():
    logits = np.zeros(8, np.float32)
    bias = np.array([0, 0, 0, 0, 1, 1, 1, 1], np.float32)
    ids, g, _ = oracle.route(logits, bias, 4)
    assert sorted(ids.tolist()) == [4, 5, 6, 7]       # bias decides the choice
    assert np.allclose(g, 0.25)                       # unbiased equal sigmoid scores


def test_router_zero_bias_is_top_logits_and_ties_go_low():
    logits, _ = synth.gen_router(32, 77, 0)
    ids, _, _ = oracle.route(logits, np.zeros(32, np.float32), 4)
    assert list(ids) == list(np.argsort(-logits.astype(np.float64), kind="stable")[:4])
    ids, g, _ = oracle.route(np.zeros(6, np.float32), np.zeros(6, np.float32), 3)
    assert list(ids) == [0, 1, 2] and np.allclose(g, 1 / 3)


# --------------------------------------------------------------------- MoE --

def _moe_inputs(n_expert=4, hidden=256, inter=512, seed=21):
    gus = synth.matrix_bytes(Q4_K, inter, hidden)
    ds = synth.matrix_bytes(Q4_K, hidden, inter)
    gate = synth.gen_blocks(Q4_K, inter * n_expert, hidden, seed, 1)
    up = synth.gen_blocks(Q4_K, inter * n_expert, hidden, seed, 2)
    down = synth.gen_blocks(Q4_K, hidden * n_expert, inter, seed, 3)
    x = synth.gen_x(1, hidden, seed, 4)[0]
    return gate, up, down, gus, ds, x


def test_silu_closed_forms():
    assert oracle.silu(0.0) == 0.0
    assert oracle.silu(40.0) == pytest.approx(40.0, rel=1e-15)
    assert abs(oracle.silu(-40.0)) < 1e-15
    assert oracle.silu(1.0) == pytest.approx(1.0 / (1.0 + math.exp(-1.0)), rel=1e-15)


def test_moe_single_expert_is_a_dense_swiglu_ffn():
    n_expert, hidden, inter = 4, 256, 512
    gate, up, down, gus, ds, x = _moe_inputs(n_expert, hidden, inter)
    e = 2
    r = oracle.moe_ffn(Q4_K, gate, up, gus, Q4_K, down, ds, n_expert, [e], [1.0], hidden, inter, x)
    G = oracle.dequant(Q4_K, gate[e * gus:(e + 1) * gus], inter, hidden).astype(np.float64)
    U = oracle.dequant(Q4_K, up[e * gus:(e + 1) * gus], inter, hidden).astype(np.float64)
    D = oracle.dequant(Q4_K, down[e * ds:(e + 1) * ds], hidden, inter).astype(np.float64)
    u = G @ x.astype(np.float64)
    v = U @ x.astype(np.float64)
    h = u / (1 + np.exp(-u)) * v
    y = D @ h
    assert np.allclose(r["u"][0], u, rtol=1e-12, atol=1e-12)
    assert np.allclose(r["v"][0], v, rtol=1e-12, atol=1e-12)
    assert np.allclose(r["y"], y, rtol=1e-10, atol=1e-10)


def test_moe_is_linear_in_g_and_order_free():
    n_expert, hidden, inter = 4, 256, 512
    gate, up, down, gus, ds, x = _moe_inputs(n_expert, hidden, inter)
    ys = [oracle.moe_ffn(Q4_K, gate, up, gus, Q4_K, down, ds, n_expert, [e], [1.0],
                         hidden, inter, x)["y"] for e in range(n_expert)]
    g = np.array([0.1, 0.2, 0.3, 0.4])
    r = oracle.moe_ffn(Q4_K, gate, up, gus, Q4_K, down, ds, n_expert, [0, 1, 2, 3], g,
                       hidden, inter, x)
    assert np.allclose(r["y"], sum(gk * yk for gk, yk in zip(g, ys)), rtol=1e-10, atol=1e-10)
    r2 = oracle.moe_ffn(Q4_K, gate, up, gus, Q4_K, down, ds, n_expert, [3, 1, 0, 2],
                        g[[3, 1, 0, 2]], hidden, inter, x)
    assert np.allclose(r2["y"], r["y"], rtol=1e-12, atol=1e-12)
    with pytest.raises(ValueError):
        oracle.moe_ffn(Q4_K, gate, up, gus, Q4_K, down, ds, n_expert, [4], [1.0],
                       hidden, inter, x)
