"""Pins of the oracle's Q4_0 and Q5_K decoders (CPU only, no GPU).

FlareLLM：纯Rust打造的浏览器端LLM推理引擎, §量化技术的全面支持 names Q4_0 and the
K-quants among the formats its engine reads; the byte layouts are the GGUF
reading restated in oracle/qmv_oracle.c.  As for the first three formats, the
oracle is pinned by per-slot round trips through the test-side encoder, the
second bit-string decoder, hand-worked blocks, closed forms, the single
rounding of the Q5_K subtraction and exact rational brute force -- so that a
field read from the wrong nibble, a fifth bit taken from the wrong bit of qh,
a dropped -8 offset or a dropped min term fails one of them.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np
import pytest

import oracle
from blockpack import decode2, f16_bits, fields_q4_0, fields_q5_k, pack_q4_0, pack_q5_k
from quantized_decode_superblocks_b200 import synth

Q4_0, Q5_K = oracle.Q4_0, oracle.Q5_K
ONE = f16_bits(1.0)
ZERO = f16_bits(0.0)


def _dequant_blocks(fmt, blocks):
    W = np.concatenate(blocks)
    n = len(blocks)
    return oracle.dequant(fmt, W, n, oracle.block_weights(fmt))


def test_block_sizes():
    assert (oracle.block_weights(Q4_0), oracle.block_bytes(Q4_0)) == (32, 18)
    assert (oracle.block_weights(Q5_K), oracle.block_bytes(Q5_K)) == (256, 176)
    # 4.5 and 5.5 bits per weight
    assert oracle.block_bytes(Q4_0) * 8 / 32 == 4.5 and oracle.block_bytes(Q5_K) * 8 / 256 == 5.5


def test_q4_0_every_position_every_value():
    blocks, expect = [], []
    for i in range(32):
        for v in range(16):
            q = [8] * 32
            q[i] = v
            blocks.append(pack_q4_0(ONE, q))
            e = np.zeros(32, np.float32)
            e[i] = v - 8
            expect.append(e)
    assert np.array_equal(_dequant_blocks(Q4_0, blocks), np.array(expect))


def test_q4_0_scale_is_applied():
    d = 0.375
    got = _dequant_blocks(Q4_0, [pack_q4_0(f16_bits(d), list(range(16)) * 2)])[0]
    assert got.tolist() == [d * (v - 8) for v in list(range(16)) * 2]


def test_q5_k_every_scale_and_min_slot_every_value():
    blocks, expect = [], []
    for j in range(8):
        for v in range(64):
            sc = [0] * 8
            sc[j] = v
            blocks.append(pack_q5_k(ONE, ZERO, sc, [0] * 8, [1] * 256))
            e = np.zeros(256, np.float32)
            e[32 * j:32 * j + 32] = v
            expect.append(e)
            m = [0] * 8
            m[j] = v
            blocks.append(pack_q5_k(ZERO, ONE, [0] * 8, m, [1] * 256))
            e = np.zeros(256, np.float32)
            e[32 * j:32 * j + 32] = -v
            expect.append(e)
    assert np.array_equal(_dequant_blocks(Q5_K, blocks), np.array(expect))


def test_q5_k_every_position_every_quant():
    blocks, expect = [], []
    for i in range(256):
        for v in range(32):
            q = [0] * 256
            q[i] = v
            blocks.append(pack_q5_k(ONE, ZERO, [1] * 8, [0] * 8, q))
            e = np.zeros(256, np.float32)
            e[i] = v
            expect.append(e)
    assert np.array_equal(_dequant_blocks(Q5_K, blocks), np.array(expect))


@pytest.mark.parametrize("fmt", [Q4_0, Q5_K])
def test_second_decoder_agrees_bit_for_bit(fmt):
    bw, bb = oracle.block_weights(fmt), oracle.block_bytes(fmt)
    W = synth.gen_blocks(fmt, 40, bw * 3, seed=21, tensor_id=fmt)
    got = oracle.dequant(fmt, W, 40, bw * 3).reshape(-1, bw)
    for k in range(W.size // bb):
        ref = decode2(fmt, W[k * bb:(k + 1) * bb])
        assert np.array_equal(got[k].view(np.uint32), ref.view(np.uint32)), k


def test_synth_fields_follow_their_distributions():
    f0 = [fields_q4_0(b) for b in synth.gen_blocks(Q4_0, 400, 32, 5, 3).reshape(400, 18)]
    q0 = np.array([f["q"] for f in f0])
    assert q0.min() == 0 and q0.max() == 15 and abs(q0.mean() - 7.5) < 0.2
    d0 = np.array([f["d"] for f in f0])
    assert d0.min() >= 1e-3 * 0.999 and d0.max() <= 2e-2 * 1.001
    f5 = [fields_q5_k(b) for b in synth.gen_blocks(Q5_K, 300, 256, 5, 4).reshape(300, 176)]
    q5 = np.array([f["q"] for f in f5])
    assert q5.min() == 0 and q5.max() == 31 and abs(q5.mean() - 15.5) < 0.2
    sc = np.array([f["sc"] + f["m"] for f in f5])
    assert sc.min() == 0 and sc.max() == 63


def test_hand_worked_q4_0_block():
    # d = 0.5, q = i % 16: weights i -> 0.5 * ((i % 16) - 8)
    q = [i % 16 for i in range(32)]
    got = _dequant_blocks(Q4_0, [pack_q4_0(f16_bits(0.5), q)])[0]
    assert got.tolist() == [-4.0, -3.5, -3.0, -2.5, -2.0, -1.5, -1.0, -0.5,
                            0.0, 0.5, 1.0, 1.5, 2.0, 2.5, 3.0, 3.5] * 2


def test_hand_worked_q5_k_block():
    # d = 1, dmin = 0.5, sc_j = j + 1, m_j = 2j, q_i = (i * 7) % 32:
    # w_i = (j + 1) * q_i - j  (0.5 * 2j)
    q = [(i * 7) % 32 for i in range(256)]
    blk = pack_q5_k(ONE, f16_bits(0.5), [j + 1 for j in range(8)], [2 * j for j in range(8)], q)
    got = _dequant_blocks(Q5_K, [blk])[0]
    assert got.tolist() == [float((i // 32 + 1) * q[i] - i // 32) for i in range(256)]
    # the fifth bits alone: every quant 16 (low nibbles zero) with sc = 1
    blk = pack_q5_k(ONE, ZERO, [1] * 8, [0] * 8, [16] * 256)
    assert np.array_equal(blk[48:176], np.zeros(128, np.uint8))
    assert np.array_equal(blk[16:48], np.full(32, 255, np.uint8))
    assert _dequant_blocks(Q5_K, [blk])[0].tolist() == [16.0] * 256


def test_q5_k_single_rounding_of_the_difference():
    # d*sc*q and dmin*m are exact in f32; their difference rounds once
    d, dmin = f16_bits(1.0 + 2.0 ** -10), f16_bits(2.0 ** -14)
    blk = pack_q5_k(d, dmin, [63] * 8, [1] * 8, [31] * 256)
    got = _dequant_blocks(Q5_K, [blk])[0]
    exact = Fraction(1 + Fraction(1, 1024)) * 63 * 31 - Fraction(1, 2 ** 14)
    assert got[0] == np.float32(float(exact))
    assert all(v == got[0] for v in got)


@pytest.mark.parametrize("Q,S,M", [(0, 5, 7), (31, 63, 0), (17, 1, 63)])
def test_q5_k_constant_fields_closed_form(Q, S, M):
    d, dmin, rows, cols = 0.0078125, 0.00390625, 3, 512
    blk = pack_q5_k(f16_bits(d), f16_bits(dmin), [S] * 8, [M] * 8, [Q] * 256)
    W = np.tile(blk, rows * cols // 256)
    x = synth.gen_x(1, cols, 17, Q)
    y, _ = oracle.qmv(Q5_K, W, rows, cols, x)
    expect = (d * S * Q - dmin * M) * float(np.sum(x.astype(np.float64)))
    assert np.allclose(y, expect, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("Q", [0, 8, 15])
def test_q4_0_constant_fields_closed_form(Q):
    d, rows, cols = 0.0625, 2, 96
    W = np.tile(pack_q4_0(f16_bits(d), [Q] * 32), rows * cols // 32)
    x = synth.gen_x(1, cols, 19, Q)
    y, _ = oracle.qmv(Q4_0, W, rows, cols, x)
    assert np.allclose(y, d * (Q - 8) * float(np.sum(x.astype(np.float64))), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("fmt,rows", [(Q4_0, 1), (Q4_0, 3), (Q5_K, 1), (Q5_K, 3)])
def test_brute_force_exact_rational(fmt, rows):
    # y and the bound from the fields in exact rational arithmetic
    bw, bb = oracle.block_weights(fmt), oracle.block_bytes(fmt)
    W = synth.gen_blocks(fmt, rows, bw, 23, fmt)
    x = synth.gen_x(2, bw, 23, 7)
    y, bound = oracle.qmv(fmt, W, rows, bw, x)
    for r in range(rows):
        blk = W[r * bb:(r + 1) * bb]
        if fmt == Q4_0:
            f = fields_q4_0(blk)
            w = [Fraction(f["d"]) * (q - 8) for q in f["q"]]
        else:
            f = fields_q5_k(blk)
            w = [Fraction(np.float32(float(Fraction(f["d"]) * f["sc"][i // 32] * f["q"][i]
                                           - Fraction(f["dmin"]) * f["m"][i // 32])).item())
                 for i in range(256)]
        for t in range(2):
            exact = sum(wi * Fraction(float(xi)) for wi, xi in zip(w, x[t]))
            mag = sum(abs(wi * Fraction(float(xi))) for wi, xi in zip(w, x[t]))
            assert abs(Fraction(y[t, r]) - exact) <= Fraction(1, 2 ** 40) * mag + Fraction(1, 10 ** 30)
            assert abs(Fraction(bound[t, r]) - mag) <= Fraction(1, 2 ** 40) * mag + Fraction(1, 10 ** 30)
