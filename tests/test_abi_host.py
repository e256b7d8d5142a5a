"""Host-side checks of the C ABI (no GPU needed): the library builds and loads,
exports every function include/qmv.h declares, and rejects bad arguments with
the documented status codes before touching a device."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

import quantized_decode_superblocks_b200 as q


ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

OK, NULL, FMT, SHAPE, ALIGN, NTOK, NSEL, CUDA, DEVICE = 0, -1, -2, -3, -4, -5, -6, -7, -8
A = 0x10000          # a fake, 16-byte aligned "device" address: never dereferenced on these paths


@pytest.fixture(scope="module")
def L():
    q.build()
    return q.lib()


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "qmv.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*([a-z_][a-z0-9_]*)\s*\(",
                       src, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(L):
    names = _declared_functions()
    assert {"qmv_f32", "qmv_batched", "moe_qmv", "moe_route", "moe_ffn", "qmv_dequant",
            "qmv_check", "qmv_strerror", "qmv_block_bytes", "qmv_block_weights"} <= set(names)
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(q.EXPORTED)


def test_block_sizes_and_strerror(L):
    assert [q.qmv_block_weights(f) for f in (0, 1, 2, 3, 4)] == [32, 256, 256, 32, 256]
    assert [q.qmv_block_bytes(f) for f in (0, 1, 2, 3, 4)] == [34, 144, 210, 18, 176]
    assert q.qmv_block_bytes(5) == 0 and q.qmv_block_weights(-1) == 0
    for s in (OK, NULL, FMT, SHAPE, ALIGN, NTOK, NSEL, CUDA, DEVICE, 42):
        assert isinstance(q.strerror(s), str) and q.strerror(s)


def qb(L, fmt=1, W=A, rows=4, cols=256, x=A, y=A, n_tok=1):
    return L.qmv_batched(fmt, W, rows, cols, x, y, n_tok, None)


def test_qmv_argument_validation(L):
    assert qb(L, W=None) == NULL and qb(L, x=None) == NULL and qb(L, y=None) == NULL
    assert qb(L, fmt=5) == FMT and qb(L, fmt=-1) == FMT
    assert qb(L, rows=0) == SHAPE and qb(L, cols=0) == SHAPE
    assert qb(L, cols=128) == SHAPE            # Q4_K needs multiples of 256
    assert qb(L, fmt=0, cols=48) == SHAPE       # Q8_0 needs multiples of 32
    assert qb(L, fmt=3, cols=48) == SHAPE       # so does Q4_0
    assert qb(L, fmt=4, cols=128) == SHAPE      # Q5_K needs multiples of 256
    assert qb(L, cols=2 ** 21) == SHAPE
    assert qb(L, n_tok=0) == NTOK and qb(L, n_tok=9) == NTOK
    assert qb(L, W=A + 8) == ALIGN and qb(L, x=A + 4) == ALIGN and qb(L, y=A + 2) == ALIGN
    assert L.qmv_f32(1, A, 4, 256, A, A + 1, None) == ALIGN
    assert L.qmv_dequant(1, A, 4, 100, A, None) == SHAPE
    assert L.qmv_dequant(1, None, 4, 256, A, None) == NULL


def test_moe_argument_validation(L):
    mat = 4 * 144

    def mq(ids=A, n_expert=8, n_sel=4, stride=mat, x_stride=0, gw=None, base=A):
        return L.moe_qmv(1, base, stride, n_expert, ids, n_sel, 4, 256, A, x_stride, gw, A, None)
    assert mq(ids=None) == NULL
    assert mq(n_sel=0) == NSEL and mq(n_sel=9) == NSEL and mq(n_expert=2, n_sel=3) == NSEL
    assert mq(n_expert=0) == NSEL and mq(n_expert=2000) == NSEL
    assert mq(stride=mat - 16) == SHAPE and mq(x_stride=-4) == SHAPE
    assert mq(stride=mat + 8) == ALIGN and mq(x_stride=3) == ALIGN and mq(base=A + 2) == ALIGN
    assert L.moe_route(A, A, 32, 0, A, A, None) == NSEL
    assert L.moe_route(A, A, 32, 9, A, A, None) == NSEL
    assert L.moe_route(A, A, 3, 4, A, A, None) == NSEL
    assert L.moe_route(None, A, 32, 4, A, A, None) == NULL

    def ffn(h=A, inter=512, n_sel=4, gus=512 * 144, ds=2 * 256 * 144):
        return L.moe_ffn(1, A, A, gus, 1, A, ds, 8, A, A, n_sel, 256, inter, A, h, A, None)
    assert ffn(h=None) == NULL and ffn(inter=300) == SHAPE and ffn(n_sel=0) == NSEL
    assert ffn(gus=16) == SHAPE and ffn(h=A + 4) == ALIGN


def test_moe_ffn_routed_argument_validation(L):
    args = [A, A, 32, 4, 1, A, A, 1792 * 8 * 144, 1, A, 2048 * 7 * 144, 2048, 1792, A, A, A, A, A, A, None]
    assert L.moe_ffn_routed(*args[:-2], None, None) == NULL          # no workspace
    bad = list(args)
    bad[3] = 9
    assert L.moe_ffn_routed(*bad) == NSEL                             # top_k above 8
    bad = list(args)
    bad[12] = 1000
    assert L.moe_ffn_routed(*bad) == SHAPE                            # inter not a multiple of 256
    bad = list(args)
    bad[18] = A + 4
    assert L.moe_ffn_routed(*bad) == ALIGN                            # workspace alignment


def test_multi_argument_validation(L):
    T = q.make_tasks([(A, 4, 256, A, A), (A, 8, 512, A, A)])
    assert L.qmv_multi(1, 1, None, 2, None) == NULL
    assert L.qmv_multi(1, 1, T, 0, None) == SHAPE
    assert L.qmv_multi(1, 0, T, 2, None) == NTOK and L.qmv_multi(1, 9, T, 2, None) == NTOK
    assert L.qmv_multi(5, 1, T, 2, None) == FMT
    bad = q.make_tasks([(A, 4, 256, A, A), (A, 8, 500, A, A)])
    assert L.qmv_multi(1, 1, bad, 2, None) == SHAPE
    bad = q.make_tasks([(A, 4, 256, A, A), (A + 8, 8, 512, A, A)])
    assert L.qmv_multi(1, 1, bad, 2, None) == ALIGN
    bad = q.make_tasks([(A, 4, 256, A, A), (A, 8, 512, None, A)])
    assert L.qmv_multi(1, 1, bad, 2, None) == NULL
    q.lib().qmv_debug_fail_next_launches(1)
    assert L.qmv_multi(1, 1, T, 2, None) == CUDA
    q.lib().qmv_debug_fail_next_launches(0)


def test_chain_argument_validation(L):
    T = q.make_tasks([(A, 4, 256, A, A), (A, 8, 512, A, A)])
    assert L.qmv_chain(1, None, 2, None) == NULL
    assert L.qmv_chain(1, T, 0, None) == SHAPE
    assert L.qmv_chain(1, T, 4097, None) == SHAPE
    assert L.qmv_chain(5, T, 2, None) == FMT
    bad = q.make_tasks([(A, 4, 256, A, A), (A, 8, 500, A, A)])
    assert L.qmv_chain(1, bad, 2, None) == SHAPE
    bad = q.make_tasks([(A, 4, 256, A, A), (A + 8, 8, 512, A, A)])
    assert L.qmv_chain(1, bad, 2, None) == ALIGN
    bad = q.make_tasks([(A, 4, 256, A, A), (A, 8, 512, A, None)])
    assert L.qmv_chain(1, bad, 2, None) == NULL
    q.lib().qmv_debug_fail_next_launches(1)
    assert L.qmv_chain(1, T, 2, None) == CUDA
    q.lib().qmv_debug_fail_next_launches(0)


def test_argmax_argument_validation(L):
    assert L.qmv_argmax(0, A, 4, 64, A, A, 1, None, None) == NULL
    assert L.qmv_argmax(0, None, 4, 64, A, A, 1, A, None) == NULL
    assert L.qmv_argmax(7, A, 4, 64, A, A, 1, A, None) == FMT
    assert L.qmv_argmax(0, A, 4, 60, A, A, 1, A, None) == SHAPE
    assert L.qmv_argmax(0, A, 0, 64, A, A, 1, A, None) == SHAPE
    assert L.qmv_argmax(0, A, 4, 64, A, A, 0, A, None) == NTOK
    assert L.qmv_argmax(0, A, 4, 64, A, A, 9, A, None) == NTOK
    assert L.qmv_argmax(0, A + 8, 4, 64, A, A, 1, A, None) == ALIGN
    assert L.qmv_argmax(0, A, 4, 64, A, A, 1, A + 2, None) == ALIGN
    # the workspace form: the same checks, then the workspace itself
    assert L.qmv_argmax_ws(0, A, 4, 64, A, A, 1, A, None, None) == NULL
    assert L.qmv_argmax_ws(0, A, 4, 64, A, A, 1, A, A + 4, None) == ALIGN
    assert L.qmv_argmax_ws(0, A, 4, 64, A, A, 9, A, A, None) == NTOK


def test_injected_launch_failure_is_reported(L):
    q.lib().qmv_debug_fail_next_launches(2)
    assert qb(L) == CUDA
    assert L.moe_route(A, A, 32, 4, A, A, None) == CUDA
    # the hook is spent; validation still comes first
    q.lib().qmv_debug_fail_next_launches(1)
    assert qb(L, n_tok=0) == NTOK
    assert qb(L) == CUDA
    q.lib().qmv_debug_fail_next_launches(0)


def test_no_device_is_an_error_not_a_fallback(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert qb(L) == DEVICE
    with pytest.raises(q.QmvError):
        q.qmv_f32(1, A, 4, 256, A, A, stream=0)


def test_python_binding_fails_loudly_without_the_library(monkeypatch, tmp_path):
    monkeypatch.setattr(q, "_lib", None)
    monkeypatch.setattr(q, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError):
        q.lib()
