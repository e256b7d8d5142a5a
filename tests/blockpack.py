"""Test-side block ENCODER and a second, bit-string DECODER (no oracle code).

The encoder places chosen integer fields into block bytes following the GGUF
layout statement (the inverse direction of the oracle's decoders), so a round
trip through the oracle pins each field's position.  The second decoder reads
the same fields by absolute bit index over the block viewed as one
little-endian bit string; it shares no structure with the oracle's loops.
"""
from __future__ import annotations

import numpy as np


def f16_bits(v: float) -> int:
    return int(np.array([v], dtype=np.float16).view(np.uint16)[0])


# ------------------------------------------------------------------ encoders

def pack_q8_0(d_bits: int, q) -> np.ndarray:
    q = [int(v) for v in q]
    assert len(q) == 32 and all(-128 <= v <= 127 for v in q)
    out = np.zeros(34, dtype=np.uint8)
    out[0], out[1] = d_bits & 0xFF, d_bits >> 8
    for i, v in enumerate(q):
        out[2 + i] = v & 0xFF
    return out


def pack_q4_k(d_bits: int, dmin_bits: int, sc, m, q) -> np.ndarray:
    sc, m, q = [int(v) for v in sc], [int(v) for v in m], [int(v) for v in q]
    assert len(sc) == 8 and len(m) == 8 and len(q) == 256
    assert all(0 <= v < 64 for v in sc + m) and all(0 <= v < 16 for v in q)
    out = np.zeros(144, dtype=np.uint8)
    out[0], out[1] = d_bits & 0xFF, d_bits >> 8
    out[2], out[3] = dmin_bits & 0xFF, dmin_bits >> 8
    s = [0] * 12
    for j in range(4):
        s[j] |= sc[j]
        s[j + 4] |= m[j]
    for j in range(4, 8):
        s[j + 4] |= (sc[j] & 15) | ((m[j] & 15) << 4)
        s[j - 4] |= (sc[j] >> 4) << 6
        s[j] |= (m[j] >> 4) << 6
    out[4:16] = s
    for c in range(4):
        for l in range(32):
            out[16 + 32 * c + l] = q[64 * c + l] | (q[64 * c + 32 + l] << 4)
    return out


def pack_q6_k(d_bits: int, scales, q) -> np.ndarray:
    scales, q = [int(v) for v in scales], [int(v) for v in q]
    assert len(scales) == 16 and len(q) == 256
    assert all(-128 <= v <= 127 for v in scales) and all(0 <= v < 64 for v in q)
    out = np.zeros(210, dtype=np.uint8)
    for h in range(2):
        for t in range(4):
            for l in range(32):
                v = q[128 * h + 32 * t + l]
                k = 64 * h + l + 32 * (t & 1)
                out[k] |= (v & 15) << (0 if t < 2 else 4)
                out[128 + 32 * h + l] |= (v >> 4) << (2 * t)
    for i, v in enumerate(scales):
        out[192 + i] = v & 0xFF
    out[208], out[209] = d_bits & 0xFF, d_bits >> 8
    return out


def pack_q4_0(d_bits: int, q) -> np.ndarray:
    q = [int(v) for v in q]
    assert len(q) == 32 and all(0 <= v < 16 for v in q)
    out = np.zeros(18, dtype=np.uint8)
    out[0], out[1] = d_bits & 0xFF, d_bits >> 8
    for i, v in enumerate(q):
        # weights 0..15 in the low nibbles of bytes 2..17, weights 16..31 in the high ones
        out[2 + (i % 16)] |= v << (4 * (i // 16))
    return out


def pack_q5_k(d_bits: int, dmin_bits: int, sc, m, q) -> np.ndarray:
    """Q5_K: the Q4_K header and scale packing, 32 bytes of fifth bits, then the
    low nibbles in the Q4_K arrangement."""
    q = [int(v) for v in q]
    assert len(q) == 256 and all(0 <= v < 32 for v in q)
    lo4 = pack_q4_k(d_bits, dmin_bits, sc, m, [v & 15 for v in q])
    out = np.zeros(176, dtype=np.uint8)
    out[0:16] = lo4[0:16]
    out[48:176] = lo4[16:144]
    for i, v in enumerate(q):
        c, r = divmod(i, 64)
        hi, l = divmod(r, 32)
        out[16 + l] |= (v >> 4) << (2 * c + hi)
    return out


# ----------------------------------------------------------- second decoder

def _bits(blk: np.ndarray, start: int, n: int) -> int:
    """Unsigned integer from n bits starting at absolute bit `start` (bit k of
    the block is bit k % 8 of byte k // 8)."""
    v = 0
    for k in range(n):
        b = start + k
        v |= ((int(blk[b // 8]) >> (b % 8)) & 1) << k
    return v


def _signed(v: int, n: int) -> int:
    return v - (1 << n) if v >= 1 << (n - 1) else v


def _half(bits: int) -> float:
    return float(np.array([bits], dtype=np.uint16).view(np.float16)[0])


def fields_q8_0(blk):
    return {"d": _half(_bits(blk, 0, 16)),
            "q": [_signed(_bits(blk, 16 + 8 * i, 8), 8) for i in range(32)]}


def fields_q4_k(blk):
    sc, m = [], []
    for j in range(8):
        if j < 4:
            sc.append(_bits(blk, 32 + 8 * j, 6))
            m.append(_bits(blk, 32 + 8 * (j + 4), 6))
        else:
            # low 4 bits from the low / high nibble of scale byte j+4, top 2 bits
            # from bits 6..7 of scale byte j-4 (sc) or j (m)
            sc.append(_bits(blk, 32 + 8 * (j + 4), 4) | (_bits(blk, 32 + 8 * (j - 4) + 6, 2) << 4))
            m.append(_bits(blk, 32 + 8 * (j + 4) + 4, 4) | (_bits(blk, 32 + 8 * j + 6, 2) << 4))
    q = []
    for i in range(256):
        c, r = divmod(i, 64)
        hi, l = divmod(r, 32)
        q.append(_bits(blk, 8 * (16 + 32 * c + l) + 4 * hi, 4))
    return {"d": _half(_bits(blk, 0, 16)), "dmin": _half(_bits(blk, 16, 16)),
            "sc": sc, "m": m, "q": q}


def fields_q6_k(blk):
    q = []
    for i in range(256):
        h, r = divmod(i, 128)
        t, l = divmod(r, 32)
        low = _bits(blk, 8 * (64 * h + l + 32 * (t % 2)) + (4 if t >= 2 else 0), 4)
        high = _bits(blk, 8 * (128 + 32 * h + l) + 2 * t, 2)
        q.append(low + 16 * high)
    return {"d": _half(_bits(blk, 8 * 208, 16)),
            "scales": [_signed(_bits(blk, 8 * (192 + k), 8), 8) for k in range(16)],
            "q": q}


def fields_q4_0(blk):
    return {"d": _half(_bits(blk, 0, 16)),
            "q": [_bits(blk, 16 + 8 * (i % 16) + 4 * (i // 16), 4) for i in range(32)]}


def fields_q5_k(blk):
    # the scale / min fields sit where Q4_K has them; the nibbles start at byte 48
    f = fields_q4_k(np.concatenate([blk[0:16], blk[48:176]]))
    q = []
    for i in range(256):
        c, r = divmod(i, 64)
        hi, l = divmod(r, 32)
        q.append(f["q"][i] + 16 * _bits(blk, 8 * (16 + l) + 2 * c + hi, 1))
    f["q"] = q
    return f


def decode2(fmt: int, blk) -> np.ndarray:
    """Second decoder: fields by bit index, then the weight formula evaluated in
    f64 and rounded once to f32 (the products are exact, see the oracle)."""
    if fmt == 0:
        f = fields_q8_0(blk)
        return np.array([f["d"] * q for q in f["q"]], dtype=np.float64).astype(np.float32)
    if fmt == 1:
        f = fields_q4_k(blk)
        return np.array([f["d"] * f["sc"][i // 32] * f["q"][i] - f["dmin"] * f["m"][i // 32]
                         for i in range(256)], dtype=np.float64).astype(np.float32)
    if fmt == 3:
        f = fields_q4_0(blk)
        return np.array([f["d"] * (q - 8) for q in f["q"]], dtype=np.float64).astype(np.float32)
    if fmt == 4:
        f = fields_q5_k(blk)
        return np.array([f["d"] * f["sc"][i // 32] * f["q"][i] - f["dmin"] * f["m"][i // 32]
                         for i in range(256)], dtype=np.float64).astype(np.float32)
    f = fields_q6_k(blk)
    return np.array([f["d"] * f["scales"][i // 16] * (f["q"][i] - 32) for i in range(256)],
                    dtype=np.float64).astype(np.float32)


# ------------------------------------------------------ vectorised encoders
# The same placements as the encoders above, for many blocks at once (the
# full-value-range GPU tests pack whole matrices).  Pinned against the
# one-block encoders by a CPU test.

def pack_q8_0_many(d_bits, q) -> np.ndarray:
    d_bits = np.asarray(d_bits, dtype=np.uint16)
    q = np.asarray(q, dtype=np.int64)
    n = d_bits.shape[0]
    assert q.shape == (n, 32) and q.min() >= -128 and q.max() <= 127
    out = np.zeros((n, 34), dtype=np.uint8)
    out[:, 0] = d_bits & 0xFF
    out[:, 1] = d_bits >> 8
    out[:, 2:] = (q & 0xFF).astype(np.uint8)
    return out.reshape(-1)


def pack_q4_k_many(d_bits, dmin_bits, sc, m, q) -> np.ndarray:
    d_bits = np.asarray(d_bits, dtype=np.uint16)
    dmin_bits = np.asarray(dmin_bits, dtype=np.uint16)
    sc, m, q = (np.asarray(a, dtype=np.int64) for a in (sc, m, q))
    n = d_bits.shape[0]
    assert sc.shape == (n, 8) and m.shape == (n, 8) and q.shape == (n, 256)
    assert sc.min() >= 0 and sc.max() < 64 and m.min() >= 0 and m.max() < 64
    assert q.min() >= 0 and q.max() < 16
    out = np.zeros((n, 144), dtype=np.int64)
    out[:, 0], out[:, 1] = d_bits & 0xFF, d_bits >> 8
    out[:, 2], out[:, 3] = dmin_bits & 0xFF, dmin_bits >> 8
    s = np.zeros((n, 12), dtype=np.int64)
    s[:, 0:4] |= sc[:, 0:4]
    s[:, 4:8] |= m[:, 0:4]
    s[:, 8:12] |= (sc[:, 4:8] & 15) | ((m[:, 4:8] & 15) << 4)
    s[:, 0:4] |= (sc[:, 4:8] >> 4) << 6
    s[:, 4:8] |= (m[:, 4:8] >> 4) << 6
    out[:, 4:16] = s
    qq = q.reshape(n, 4, 2, 32)                  # [chunk c][low / high nibble][l]
    out[:, 16:] = (qq[:, :, 0, :] | (qq[:, :, 1, :] << 4)).reshape(n, 128)
    return out.astype(np.uint8).reshape(-1)


def pack_q6_k_many(d_bits, scales, q) -> np.ndarray:
    d_bits = np.asarray(d_bits, dtype=np.uint16)
    scales, q = np.asarray(scales, dtype=np.int64), np.asarray(q, dtype=np.int64)
    n = d_bits.shape[0]
    assert scales.shape == (n, 16) and q.shape == (n, 256)
    assert scales.min() >= -128 and scales.max() <= 127 and q.min() >= 0 and q.max() < 64
    out = np.zeros((n, 210), dtype=np.int64)
    qq = q.reshape(n, 2, 4, 32)                  # [half h][t][l]
    for h in range(2):
        for t in range(4):
            k0 = 64 * h + 32 * (t & 1)
            out[:, k0:k0 + 32] |= (qq[:, h, t, :] & 15) << (0 if t < 2 else 4)
            out[:, 128 + 32 * h:160 + 32 * h] |= (qq[:, h, t, :] >> 4) << (2 * t)
    out[:, 192:208] = scales & 0xFF
    out[:, 208], out[:, 209] = d_bits & 0xFF, d_bits >> 8
    return out.astype(np.uint8).reshape(-1)


def pack_q4_0_many(d_bits, q) -> np.ndarray:
    d_bits = np.asarray(d_bits, dtype=np.uint16)
    q = np.asarray(q, dtype=np.int64)
    n = d_bits.shape[0]
    assert q.shape == (n, 32) and q.min() >= 0 and q.max() < 16
    out = np.zeros((n, 18), dtype=np.int64)
    out[:, 0], out[:, 1] = d_bits & 0xFF, d_bits >> 8
    out[:, 2:] = q[:, :16] | (q[:, 16:] << 4)
    return out.astype(np.uint8).reshape(-1)


def pack_q5_k_many(d_bits, dmin_bits, sc, m, q) -> np.ndarray:
    q = np.asarray(q, dtype=np.int64)
    n = q.shape[0]
    assert q.shape == (n, 256) and q.min() >= 0 and q.max() < 32
    lo4 = pack_q4_k_many(d_bits, dmin_bits, sc, m, q & 15).reshape(n, 144)
    out = np.zeros((n, 176), dtype=np.int64)
    out[:, 0:16] = lo4[:, 0:16]
    out[:, 48:176] = lo4[:, 16:144]
    qq = (q >> 4).reshape(n, 4, 2, 32)            # [chunk c][low / high nibble][l]
    for c in range(4):
        for hi in range(2):
            out[:, 16:48] |= qq[:, c, hi, :] << (2 * c + hi)
    return out.astype(np.uint8).reshape(-1)
