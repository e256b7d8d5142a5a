"""quantized_decode_superblocks_b200 -- Python binding of libqmv.so.

The decode-step matvec of GGUF block-quantized weights (Q8_0, Q4_0, Q4_K, Q5_K,
Q6_K) with f32 activations, dequantized on the fly, on an NVIDIA B200 (sm_100a).  Every
step runs in the library's CUDA kernels; this module only marshals arguments
(tensor data pointers, sizes, the current CUDA stream) through ctypes to the C
ABI declared in ``include/qmv.h``, with the same function names.  PyTorch
provides device memory and streams.  There is no CPU fallback: if the library
is missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os

from .synth import Q4_0, Q4_K, Q5_K, Q6_K, Q8_0  # noqa: F401  (format ids)

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqmv.so")

QMV_OK = 0
STATUS_NAMES = {0: "QMV_OK", -1: "QMV_ERR_NULL", -2: "QMV_ERR_FMT", -3: "QMV_ERR_SHAPE",
                -4: "QMV_ERR_ALIGN", -5: "QMV_ERR_NTOK", -6: "QMV_ERR_NSEL", -7: "QMV_ERR_CUDA",
                -8: "QMV_ERR_DEVICE"}
DEVERR_EXPERT_ID = 1
DEVERR_TIMEOUT = 2
DEVERR_DRAIN = 4
KERNEL_WARP_RING, KERNEL_GENERAL, KERNEL_TENSOR_CORE, KERNEL_STREAM = 1, 2, 3, 4

EXPORTED = ("qmv_f32", "qmv_batched", "qmv_multi", "qmv_chain", "qmv_argmax", "qmv_argmax_ws", "moe_route", "moe_qmv", "moe_ffn", "moe_ffn_routed", "moe_ffn_static",
            "qmv_dequant",
            "qmv_check", "qmv_strerror", "qmv_block_bytes", "qmv_block_weights",
            "qmv_debug_fail_next_launches", "qmv_debug_short_copies", "qmv_set_pdl", "qmv_get_pdl",
            "qmv_last_cuda_error", "qmv_debug_last_kernel")


class QmvTask(ctypes.Structure):
    """One matvec of a grouped launch (qmv_task in include/qmv.h)."""
    _fields_ = [("W_blocks", ctypes.c_void_p), ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("x", ctypes.c_void_p), ("y", ctypes.c_void_p)]


class QmvError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = strerror(status)
        if status == -7:
            detail += ": " + lib().qmv_last_cuda_error().decode()
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} ({detail})")


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libqmv.so (built by ``build()``); raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built: run quantized_decode_superblocks_b200.build()")
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, c_int = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        L.qmv_f32.argtypes = [c_int, vp, i64, i64, vp, vp, vp]
        L.qmv_batched.argtypes = [c_int, vp, i64, i64, vp, vp, c_int, vp]
        L.qmv_multi.argtypes = [c_int, c_int, ctypes.POINTER(QmvTask), c_int, vp]
        L.qmv_chain.argtypes = [c_int, ctypes.POINTER(QmvTask), c_int, vp]
        L.qmv_argmax.argtypes = [c_int, vp, i64, i64, vp, vp, c_int, vp, vp]
        L.qmv_argmax_ws.argtypes = [c_int, vp, i64, i64, vp, vp, c_int, vp, vp, vp]
        L.moe_route.argtypes = [vp, vp, c_int, c_int, vp, vp, vp]
        L.moe_qmv.argtypes = [c_int, vp, i64, c_int, vp, c_int, i64, i64, vp, i64, vp, vp, vp]
        L.moe_ffn.argtypes = [c_int, vp, vp, i64, c_int, vp, i64, c_int, vp, vp, c_int, i64, i64,
                              vp, vp, vp, vp]
        L.moe_ffn_routed.argtypes = [vp, vp, c_int, c_int, c_int, vp, vp, i64, c_int, vp, i64, i64, i64,
                                     vp, vp, vp, vp, vp, vp, vp]
        L.moe_ffn_static.argtypes = [c_int, vp, vp, i64, c_int, vp, i64, c_int, vp, vp, c_int, i64, i64,
                                     vp, vp, vp]
        L.qmv_dequant.argtypes = [c_int, vp, i64, i64, vp, vp]
        L.qmv_check.argtypes = [vp, ctypes.POINTER(c_int)]
        L.qmv_strerror.argtypes = [c_int]
        L.qmv_strerror.restype = ctypes.c_char_p
        L.qmv_block_bytes.argtypes = [c_int]
        L.qmv_block_bytes.restype = ctypes.c_size_t
        L.qmv_block_weights.argtypes = [c_int]
        L.qmv_debug_fail_next_launches.argtypes = [c_int]
        L.qmv_debug_fail_next_launches.restype = None
        L.qmv_debug_short_copies.argtypes = [c_int]
        L.qmv_debug_short_copies.restype = None
        L.qmv_set_pdl.argtypes = [c_int]
        L.qmv_set_pdl.restype = None
        L.qmv_get_pdl.argtypes = []
        L.qmv_debug_last_kernel.argtypes = []
        L.qmv_last_cuda_error.argtypes = []
        L.qmv_last_cuda_error.restype = ctypes.c_char_p
        for name in EXPORTED:
            if name not in ("qmv_strerror", "qmv_block_bytes", "qmv_debug_fail_next_launches",
                            "qmv_debug_short_copies", "qmv_set_pdl", "qmv_last_cuda_error"):
                getattr(L, name).restype = c_int
        _lib = L
    return _lib


def build(verbose: bool = False) -> str:
    from .buildlib import build as _build
    return _build(verbose=verbose)


def strerror(status: int) -> str:
    return lib().qmv_strerror(status).decode()


def _ptr(t) -> int:
    """Device (or host) address of a tensor, an int address, or None -> NULL."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int, where: str):
    if rc != QMV_OK:
        raise QmvError(rc, where)


def qmv_set_pdl(enable: bool) -> None:
    """Programmatic dependent launch for matvec launches (see include/qmv.h)."""
    lib().qmv_set_pdl(1 if enable else 0)


def qmv_get_pdl() -> bool:
    return bool(lib().qmv_get_pdl())


def qmv_debug_last_kernel() -> int:
    """Which kernel served this thread's most recent matvec call (KERNEL_*)."""
    return lib().qmv_debug_last_kernel()


def qmv_block_bytes(fmt: int) -> int:
    return lib().qmv_block_bytes(fmt)


def qmv_block_weights(fmt: int) -> int:
    return lib().qmv_block_weights(fmt)


def qmv_f32(fmt, W, rows, cols, x, y, stream=None):
    """y[rows] = W x (see include/qmv.h)."""
    _check(lib().qmv_f32(fmt, _ptr(W), rows, cols, _ptr(x), _ptr(y), _stream(stream)), "qmv_f32")


def qmv_batched(fmt, W, rows, cols, x, y, n_tok, stream=None):
    """y[n_tok][rows] = W x[n_tok][cols]^T, 1 <= n_tok <= 8."""
    _check(lib().qmv_batched(fmt, _ptr(W), rows, cols, _ptr(x), _ptr(y), n_tok, _stream(stream)),
           "qmv_batched")


def make_tasks(tasks):
    """ctypes array of QmvTask from (W, rows, cols, x, y) tuples."""
    arr = (QmvTask * len(tasks))()
    for i, (W, rows, cols, x, y) in enumerate(tasks):
        arr[i] = QmvTask(_ptr(W), rows, cols, _ptr(x), _ptr(y))
    return arr


def qmv_multi(fmt, n_tok, tasks, stream=None):
    """Independent matvecs y_t = W_t x_t in grouped launches; `tasks` is a list of
    (W, rows, cols, x, y) tuples or an array from make_tasks()."""
    arr = tasks if isinstance(tasks, ctypes.Array) else make_tasks(tasks)
    _check(lib().qmv_multi(fmt, n_tok, arr, len(arr), _stream(stream)), "qmv_multi")


def qmv_chain(fmt, tasks, stream=None):
    """One-token matvecs executed in order (task t+1 may read task t's y);
    `tasks` as for qmv_multi."""
    arr = tasks if isinstance(tasks, ctypes.Array) else make_tasks(tasks)
    _check(lib().qmv_chain(fmt, arr, len(arr), _stream(stream)), "qmv_chain")


def qmv_argmax(fmt, W, rows, cols, x, y, n_tok, idx_out, stream=None):
    """y = W x (kept in y) and idx_out[t] = argmax over rows of y[t] (ties to the
    lower row, NaN skipped, -1 if all NaN)."""
    _check(lib().qmv_argmax(fmt, _ptr(W), rows, cols, _ptr(x), _ptr(y), n_tok, _ptr(idx_out),
                            _stream(stream)), "qmv_argmax")


ARGMAX_WS_BYTES = 128


def qmv_argmax_ws(fmt, W, rows, cols, x, y, n_tok, idx_out, workspace, stream=None):
    """qmv_argmax with a caller-owned workspace of ARGMAX_WS_BYTES device bytes
    (zero before the first call; every completed call leaves it zero)."""
    _check(lib().qmv_argmax_ws(fmt, _ptr(W), rows, cols, _ptr(x), _ptr(y), n_tok, _ptr(idx_out),
                               _ptr(workspace), _stream(stream)), "qmv_argmax_ws")


def moe_route(logits, bias, n_expert, top_k, ids_out, g_out, stream=None):
    _check(lib().moe_route(_ptr(logits), _ptr(bias), n_expert, top_k, _ptr(ids_out), _ptr(g_out),
                           _stream(stream)), "moe_route")


def moe_qmv(fmt, expert_blocks, expert_stride_bytes, n_expert, expert_ids, n_sel, rows, cols,
            x, x_stride, gate_w, y, stream=None):
    _check(lib().moe_qmv(fmt, _ptr(expert_blocks), expert_stride_bytes, n_expert, _ptr(expert_ids),
                         n_sel, rows, cols, _ptr(x), x_stride, _ptr(gate_w), _ptr(y),
                         _stream(stream)), "moe_qmv")


def moe_ffn(fmt_gu, gate_blocks, up_blocks, gu_stride_bytes, fmt_down, down_blocks,
            down_stride_bytes, n_expert, expert_ids, g, n_sel, hidden, inter, x, h_scratch, y,
            stream=None):
    _check(lib().moe_ffn(fmt_gu, _ptr(gate_blocks), _ptr(up_blocks), gu_stride_bytes, fmt_down,
                         _ptr(down_blocks), down_stride_bytes, n_expert, _ptr(expert_ids), _ptr(g),
                         n_sel, hidden, inter, _ptr(x), _ptr(h_scratch), _ptr(y), _stream(stream)),
           "moe_ffn")


MOE_WS_BYTES = 16


def moe_ffn_routed(logits, bias, n_expert, top_k, fmt_gu, gate_blocks, up_blocks, gu_stride_bytes,
                   fmt_down, down_blocks, down_stride_bytes, hidden, inter, x, ids_out, g_out, h_scratch, y,
                   workspace, stream=None):
    """Router + MoE FFN step (one launch where the shapes allow; see include/qmv.h)."""
    _check(lib().moe_ffn_routed(_ptr(logits), _ptr(bias), n_expert, top_k, fmt_gu, _ptr(gate_blocks),
                                _ptr(up_blocks), gu_stride_bytes, fmt_down, _ptr(down_blocks), down_stride_bytes,
                                hidden, inter, _ptr(x), _ptr(ids_out), _ptr(g_out), _ptr(h_scratch), _ptr(y),
                                _ptr(workspace), _stream(stream)), "moe_ffn_routed")


def moe_ffn_static(fmt_gu, gate_blocks, up_blocks, gu_stride_bytes, fmt_down, down_blocks,
                   down_stride_bytes, n_expert, expert_ids, g, n_sel, hidden, inter, x, y, stream=None):
    """moe_ffn with the library's own fixed device scratch (see include/qmv.h)."""
    _check(lib().moe_ffn_static(fmt_gu, _ptr(gate_blocks), _ptr(up_blocks), gu_stride_bytes, fmt_down,
                                _ptr(down_blocks), down_stride_bytes, n_expert, _ptr(expert_ids), _ptr(g),
                                n_sel, hidden, inter, _ptr(x), _ptr(y), _stream(stream)), "moe_ffn_static")


def qmv_dequant(fmt, W, rows, cols, out, stream=None):
    _check(lib().qmv_dequant(fmt, _ptr(W), rows, cols, _ptr(out), _stream(stream)), "qmv_dequant")


def qmv_check(stream=None) -> int:
    """Synchronises the stream; returns the device error bits (0 = none).
    Raises QmvError only when the synchronisation itself fails."""
    word = ctypes.c_int(0)
    rc = lib().qmv_check(_stream(stream), ctypes.byref(word))
    if rc not in (QMV_OK, -8):
        raise QmvError(rc, "qmv_check")
    return word.value
