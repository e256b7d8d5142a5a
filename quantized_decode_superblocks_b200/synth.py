"""Seeded synthetic inputs in GGUF block layout: weights, activations, router.

This module holds NONE of the method's arithmetic: it never decodes a block.
It fills each block's bytes so that every field follows its stated
distribution, using a counter-based generator (numpy's Philox keyed by
(seed, tensor_id)), so any tensor can be regenerated from its two keys.  Both
the tests' oracle side and the CUDA side take their inputs from here.

Field byte ranges per block (GGUF layout, little-endian):
  Q8_0 (34 B):  [0,2) fp16 d ~ U[1e-3, 2e-2];  [2,34) int8 q ~ U{-127..127}.
  Q4_K (144 B): [0,2) fp16 d, [2,4) fp16 dmin, both ~ U[1e-3, 1e-2];
                [4,16) packed 6-bit scales/mins and [16,144) packed nibbles:
                uniform random bytes.  The 12 scale bytes carry exactly sixteen
                6-bit fields (96 bits, a bijection) and each quant byte two
                nibbles, so uniform bytes give independent sc, m ~ U{0..63} and
                q ~ U{0..15}.
  Q6_K (210 B): [0,192) ql / qh: uniform random bytes, so the 6-bit quants are
                U{0..63}; [192,208) int8 scales ~ U{-64..63};
                [208,210) fp16 d ~ U[1e-4, 2e-3].
  Q4_0 (18 B):  [0,2) fp16 d ~ U[1e-3, 2e-2]; [2,18) packed nibbles: uniform
                random bytes, so q ~ U{0..15}.
  Q5_K (176 B): [0,2) fp16 d, [2,4) fp16 dmin, both ~ U[1e-3, 1e-2];
                [4,16) scales, [16,48) fifth bits, [48,176) nibbles: uniform
                random bytes, so sc, m ~ U{0..63} and q ~ U{0..31}.
No page or workload fixes distributions for Q4_0 and Q5_K; these mirror Q8_0
and Q4_K.
Uniform reals are drawn in f64 and rounded to fp16 by numpy (round to nearest
even).  Activations and router logits are f32 N(0, 1); the expert bias is
f32 N(0, 0.1).
"""
from __future__ import annotations

import numpy as np

Q8_0, Q4_K, Q6_K, Q4_0, Q5_K = 0, 1, 2, 3, 4
FORMAT_NAMES = {Q8_0: "Q8_0", Q4_K: "Q4_K", Q6_K: "Q6_K", Q4_0: "Q4_0", Q5_K: "Q5_K"}
BLOCK_WEIGHTS = {Q8_0: 32, Q4_K: 256, Q6_K: 256, Q4_0: 32, Q5_K: 256}
BLOCK_BYTES = {Q8_0: 34, Q4_K: 144, Q6_K: 210, Q4_0: 18, Q5_K: 176}


def rng(seed: int, tensor_id: int) -> np.random.Generator:
    key = np.array([seed & 0xFFFFFFFFFFFFFFFF, tensor_id & 0xFFFFFFFFFFFFFFFF], dtype=np.uint64)
    return np.random.Generator(np.random.Philox(key=key))


def matrix_bytes(fmt: int, rows: int, cols: int) -> int:
    assert cols % BLOCK_WEIGHTS[fmt] == 0
    return rows * (cols // BLOCK_WEIGHTS[fmt]) * BLOCK_BYTES[fmt]


def _fp16_uniform(g: np.random.Generator, n: int, lo: float, hi: float) -> np.ndarray:
    return g.uniform(lo, hi, size=n).astype(np.float16).view(np.uint8).reshape(n, 2)


def gen_blocks(fmt: int, rows: int, cols: int, seed: int, tensor_id: int) -> np.ndarray:
    """uint8 array of rows * (cols / bw) blocks, dense row-major, no padding."""
    bw, bb = BLOCK_WEIGHTS[fmt], BLOCK_BYTES[fmt]
    if cols % bw or rows < 1:
        raise ValueError(f"{FORMAT_NAMES[fmt]}: cols must be a positive multiple of {bw}")
    nblk = rows * (cols // bw)
    g = rng(seed, tensor_id)
    buf = np.frombuffer(g.bytes(nblk * bb), dtype=np.uint8).reshape(nblk, bb).copy()
    if fmt == Q8_0:
        buf[:, 0:2] = _fp16_uniform(g, nblk, 1e-3, 2e-2)
        q = g.integers(-127, 128, size=(nblk, 32), dtype=np.int8)
        buf[:, 2:34] = q.view(np.uint8)
    elif fmt == Q4_K:
        buf[:, 0:2] = _fp16_uniform(g, nblk, 1e-3, 1e-2)
        buf[:, 2:4] = _fp16_uniform(g, nblk, 1e-3, 1e-2)
    elif fmt == Q6_K:
        sc = g.integers(-64, 64, size=(nblk, 16), dtype=np.int8)
        buf[:, 192:208] = sc.view(np.uint8)
        buf[:, 208:210] = _fp16_uniform(g, nblk, 1e-4, 2e-3)
    elif fmt == Q4_0:
        buf[:, 0:2] = _fp16_uniform(g, nblk, 1e-3, 2e-2)
    elif fmt == Q5_K:
        buf[:, 0:2] = _fp16_uniform(g, nblk, 1e-3, 1e-2)
        buf[:, 2:4] = _fp16_uniform(g, nblk, 1e-3, 1e-2)
    else:
        raise ValueError("unknown format")
    return buf.reshape(-1)


def gen_x(n_tok: int, cols: int, seed: int, tensor_id: int) -> np.ndarray:
    """f32 activations [n_tok, cols] ~ N(0, 1)."""
    return rng(seed, tensor_id).standard_normal((n_tok, cols), dtype=np.float32)


def gen_router(n_expert: int, seed: int, tensor_id: int):
    """(logits ~ N(0,1), bias ~ N(0, 0.1)), both f32 [n_expert]."""
    g = rng(seed, tensor_id)
    logits = g.standard_normal(n_expert, dtype=np.float32)
    bias = (g.standard_normal(n_expert, dtype=np.float64) * 0.1).astype(np.float32)
    return logits, bias


# ------------------------------------------------------------------ workloads
# Shapes and seeds of the measured workloads.  Each is synthetic: the real
# model files the pages speak of are not available, so these stand in for them.

def workload_cfg0():
    """Q8_0 1024 x 1024, one token, seed 0."""
    return dict(fmt=Q8_0, rows=1024, cols=1024, n_tok=1, seed=0)


def workload_cfg1():
    """Q4_K fused QKV 3072 x 2048 (Q 2048 + K 512 + V 512 rows: 32 query heads and
    8 KV heads of head_dim 64), one token."""
    return dict(fmt=Q4_K, rows=3072, cols=2048, n_tok=1, seed=1,
                segments=[("q", 0, 2048), ("k", 2048, 2560), ("v", 2560, 3072)])


def workload_cfg2(n_tok: int = 1):
    """Q6_K output / vocab projection 128000 x 2048, n_tok in {1, 4}."""
    return dict(fmt=Q6_K, rows=128000, cols=2048, n_tok=n_tok, seed=2)


def workload_cfg3():
    """MoE: 32 experts, Q4_K gate / up [1792 x 2048] and down [2048 x 1792], top-4."""
    return dict(fmt=Q4_K, n_expert=32, top_k=4, hidden=2048, inter=1792, seed=3)


def workload_cfg4_layer():
    """One layer of the 16-layer Q8_0 dense stack (hidden 2048, intermediate 8192,
    32 / 8 heads, head_dim 64): (name, rows, cols) of its four matvecs."""
    return [("qkv", 3072, 2048), ("o", 2048, 2048), ("gate_up", 16384, 2048), ("down", 2048, 8192)]


CFG4_LAYERS = 16
CFG4_SEED = 4

LFM_LAYERS = 24
LFM_SEED = 5


def lfm_attention_layer(layer: int) -> bool:
    """Six of the 24 layers are attention layers, spread evenly: every fourth,
    from layer 3 (the pages say only that they are sparsely distributed)."""
    return layer % 4 == 3


def workload_lfm_mix():
    """One decode token of an LFM2.5-style decoder (BebeLM：纯Rust实现的端侧大模型
    推理引擎, §独特的层设计, §门控短卷积, §量化格式支持, §核心算子): hidden 2048,
    24 layers -- 6 GQA attention layers (32 query / 8 KV heads of 64) and 18
    gated short-convolution layers -- each followed by a top-4-of-32 MoE FFN,
    then the 128000-row vocabulary projection with greedy argmax.  Weights are
    Q4_K except the sensitive tensors the page names, which are Q6_K (the
    attention V projection and the vocabulary).  The weight matvecs of one
    layer kind, in order, as (name, fmt, rows, cols):"""
    return dict(
        attention=[("qk", Q4_K, 2560, 2048), ("v", Q6_K, 512, 2048), ("o", Q4_K, 2048, 2048)],
        conv=[("in_proj", Q4_K, 3 * 2048, 2048), ("out_proj", Q4_K, 2048, 2048)],
        moe=dict(fmt=Q4_K, n_expert=32, top_k=4, hidden=2048, inter=1792),
        vocab=(Q6_K, 128000, 2048), layers=LFM_LAYERS, seed=LFM_SEED)
