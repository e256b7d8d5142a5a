"""The oracle: a plain, slow CPU restatement of the quantized decode matvec.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  The CUDA
library never links, imports or calls it, and shares no code with it.

The arithmetic lives in ``qmv_oracle.c`` (plain C, f64 accumulation, built with
``-ffp-contract=off``); this module only marshals numpy arrays through ctypes.
See ``qmv_oracle.h`` for what each function computes and the passages it follows.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from .build import build_oracle, library_path

Q8_0, Q4_K, Q6_K, Q4_0, Q5_K = 0, 1, 2, 3, 4

_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        path = library_path()
        if not os.path.exists(path) or _stale(path):
            build_oracle()
        L = ctypes.CDLL(path)
        u8p = ctypes.POINTER(ctypes.c_uint8)
        f32p = ctypes.POINTER(ctypes.c_float)
        f64p = ctypes.POINTER(ctypes.c_double)
        i32p = ctypes.POINTER(ctypes.c_int32)
        i64p = ctypes.POINTER(ctypes.c_int64)
        i64 = ctypes.c_int64
        c_int = ctypes.c_int
        L.orc_half_to_float.argtypes = [ctypes.c_uint16]
        L.orc_half_to_float.restype = ctypes.c_float
        L.orc_block_weights.argtypes = [c_int]
        L.orc_block_bytes.argtypes = [c_int]
        for name in ("orc_dequant_block_q8_0", "orc_dequant_block_q4_k", "orc_dequant_block_q6_k",
                     "orc_dequant_block_q4_0", "orc_dequant_block_q5_k"):
            getattr(L, name).argtypes = [u8p, f32p]
            getattr(L, name).restype = None
        L.orc_dequant.argtypes = [c_int, u8p, i64, i64, f32p]
        L.orc_qmv.argtypes = [c_int, u8p, i64, i64, f32p, c_int, f64p, f64p, c_int]
        L.orc_qmv_rows.argtypes = [c_int, u8p, i64, i64, i64p, i64, f32p, c_int, f64p, f64p]
        L.orc_route.argtypes = [f32p, f32p, c_int, c_int, i32p, f64p, f32p]
        L.orc_silu.argtypes = [ctypes.c_double]
        L.orc_silu.restype = ctypes.c_double
        L.orc_moe_ffn.argtypes = [c_int, u8p, u8p, i64, c_int, u8p, i64, c_int, i32p, f64p,
                                  c_int, i64, i64, f32p, f64p, f64p, f64p, f64p]
        _lib = L
    return _lib


def _stale(path: str) -> bool:
    here = os.path.dirname(os.path.abspath(__file__))
    so_t = os.path.getmtime(path)
    return any(os.path.getmtime(os.path.join(here, f)) > so_t
               for f in ("qmv_oracle.c", "qmv_oracle.h"))


def _p(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _null(ctype):
    return ctypes.POINTER(ctype)()


def block_weights(fmt: int) -> int:
    return lib().orc_block_weights(fmt)


def block_bytes(fmt: int) -> int:
    return lib().orc_block_bytes(fmt)


def half_to_float(bits: int) -> float:
    return lib().orc_half_to_float(bits)


def dequant_block(fmt: int, blk: np.ndarray) -> np.ndarray:
    blk = np.ascontiguousarray(blk, dtype=np.uint8)
    assert blk.size == block_bytes(fmt)
    out = np.empty(block_weights(fmt), dtype=np.float32)
    fn = {Q8_0: lib().orc_dequant_block_q8_0, Q4_K: lib().orc_dequant_block_q4_k,
          Q6_K: lib().orc_dequant_block_q6_k, Q4_0: lib().orc_dequant_block_q4_0,
          Q5_K: lib().orc_dequant_block_q5_k}[fmt]
    fn(_p(blk, ctypes.c_uint8), _p(out, ctypes.c_float))
    return out


def dequant(fmt: int, W: np.ndarray, rows: int, cols: int) -> np.ndarray:
    W = np.ascontiguousarray(W, dtype=np.uint8)
    out = np.empty((rows, cols), dtype=np.float32)
    rc = lib().orc_dequant(fmt, _p(W, ctypes.c_uint8), rows, cols, _p(out, ctypes.c_float))
    if rc != 0:
        raise ValueError("orc_dequant: bad arguments")
    return out


def qmv(fmt: int, W: np.ndarray, rows: int, cols: int, x: np.ndarray, nthreads: int = 1):
    """Returns (y, bound), both float64 [n_tok, rows]; x is [n_tok, cols] or [cols]."""
    W = np.ascontiguousarray(W, dtype=np.uint8)
    x2 = np.ascontiguousarray(np.atleast_2d(x), dtype=np.float32)
    n_tok = x2.shape[0]
    assert x2.shape[1] == cols
    y = np.empty((n_tok, rows), dtype=np.float64)
    b = np.empty((n_tok, rows), dtype=np.float64)
    rc = lib().orc_qmv(fmt, _p(W, ctypes.c_uint8), rows, cols, _p(x2, ctypes.c_float), n_tok,
                       _p(y, ctypes.c_double), _p(b, ctypes.c_double), nthreads)
    if rc != 0:
        raise ValueError("orc_qmv: bad arguments")
    return y, b


def qmv_rows(fmt: int, W: np.ndarray, rows: int, cols: int, row_idx, x: np.ndarray):
    """(y, bound) for the listed rows only: float64 [n_tok, len(row_idx)]."""
    W = np.ascontiguousarray(W, dtype=np.uint8)
    idx = np.ascontiguousarray(row_idx, dtype=np.int64)
    x2 = np.ascontiguousarray(np.atleast_2d(x), dtype=np.float32)
    n_tok = x2.shape[0]
    y = np.empty((n_tok, idx.size), dtype=np.float64)
    b = np.empty((n_tok, idx.size), dtype=np.float64)
    rc = lib().orc_qmv_rows(fmt, _p(W, ctypes.c_uint8), rows, cols, _p(idx, ctypes.c_int64),
                            idx.size, _p(x2, ctypes.c_float), n_tok,
                            _p(y, ctypes.c_double), _p(b, ctypes.c_double))
    if rc != 0:
        raise ValueError("orc_qmv_rows: bad arguments")
    return y, b


def route(logits: np.ndarray, bias: np.ndarray, top_k: int):
    """Returns (ids int32[top_k], g float64[top_k], biased float32[n_expert])."""
    lg = np.ascontiguousarray(logits, dtype=np.float32)
    bs = np.ascontiguousarray(bias, dtype=np.float32)
    n = lg.size
    ids = np.empty(top_k, dtype=np.int32)
    g = np.empty(top_k, dtype=np.float64)
    biased = np.empty(n, dtype=np.float32)
    rc = lib().orc_route(_p(lg, ctypes.c_float), _p(bs, ctypes.c_float), n, top_k,
                         _p(ids, ctypes.c_int32), _p(g, ctypes.c_double),
                         _p(biased, ctypes.c_float))
    if rc != 0:
        raise ValueError("orc_route: bad arguments")
    return ids, g, biased


def silu(z: float) -> float:
    return lib().orc_silu(z)


def moe_ffn(fmt_gu: int, gate_all: np.ndarray, up_all: np.ndarray, gu_stride: int,
            fmt_down: int, down_all: np.ndarray, down_stride: int, n_expert: int,
            ids: np.ndarray, g: np.ndarray, hidden: int, inter: int, x: np.ndarray):
    """Returns dict(u, v, h [n_sel, inter], y [hidden]) in float64."""
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    g = np.ascontiguousarray(g, dtype=np.float64)
    x = np.ascontiguousarray(x, dtype=np.float32)
    gate_all = np.ascontiguousarray(gate_all, dtype=np.uint8)
    up_all = np.ascontiguousarray(up_all, dtype=np.uint8)
    down_all = np.ascontiguousarray(down_all, dtype=np.uint8)
    n_sel = ids.size
    u = np.empty((n_sel, inter)); v = np.empty((n_sel, inter)); h = np.empty((n_sel, inter))
    y = np.empty(hidden)
    rc = lib().orc_moe_ffn(fmt_gu, _p(gate_all, ctypes.c_uint8), _p(up_all, ctypes.c_uint8),
                           gu_stride, fmt_down, _p(down_all, ctypes.c_uint8), down_stride,
                           n_expert, _p(ids, ctypes.c_int32), _p(g, ctypes.c_double), n_sel,
                           hidden, inter, _p(x, ctypes.c_float), _p(u, ctypes.c_double),
                           _p(v, ctypes.c_double), _p(h, ctypes.c_double), _p(y, ctypes.c_double))
    if rc != 0:
        raise ValueError("orc_moe_ffn: bad arguments")
    return {"u": u, "v": v, "h": h, "y": y}
