"""moe_ffn_static -- the MoE FFN step for callers that cannot allocate device
memory (e.g. code running inside a CUDA-graph capture, or a plugin handed only
its input and output buffers).  Its SwiGLU scratch is the library's own
fixed-size device array instead of a caller buffer.

Checked through the C ABI against moe_ffn (the entry point with a caller
scratch buffer) on the same inputs, on two calls in a row: both run the same
kernels in the same order on the same values, so the outputs must agree bit
for bit (tighter than the matvec tolerance the other tests use).  This file is collected last so that a run that
stops at the first failure has run every other test before it."""
from __future__ import annotations

import numpy as np
import pytest

import quantized_decode_superblocks_b200 as q
from quantized_decode_superblocks_b200 import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

Q4_K = synth.Q4_K


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def test_moe_ffn_static_matches_moe_ffn_on_two_calls():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    q.build()
    E, hidden, inter, seed = 8, 1024, 1792, 91
    gus = synth.matrix_bytes(Q4_K, inter, hidden)
    ds = synth.matrix_bytes(Q4_K, hidden, inter)
    gate = dev(synth.gen_blocks(Q4_K, inter * E, hidden, seed, 1))
    up = dev(synth.gen_blocks(Q4_K, inter * E, hidden, seed, 2))
    down = dev(synth.gen_blocks(Q4_K, hidden * E, inter, seed, 3))
    cases = [([3, 6, 0, 5], [0.4, 0.3, 0.2, 0.1]), ([7, 1, 2, 4, 5, 0], [0.1, 0.2, 0.1, 0.3, 0.2, 0.1])]
    for call, (ids, g) in enumerate(cases):
        n_sel = len(ids)
        ids_d = dev(np.array(ids, np.int32))
        g_d = dev(np.array(g, np.float32))
        x = dev(synth.gen_x(1, hidden, seed, 10 + call)[0])
        h = torch.empty((n_sel, inter), device="cuda")
        y_ref = torch.empty(hidden, device="cuda")
        y = torch.full((hidden,), float("nan"), device="cuda")
        q.moe_ffn(Q4_K, gate, up, gus, Q4_K, down, ds, E, ids_d, g_d, n_sel, hidden, inter, x, h, y_ref)
        q.moe_ffn_static(Q4_K, gate, up, gus, Q4_K, down, ds, E, ids_d, g_d, n_sel, hidden, inter, x, y)
        torch.cuda.synchronize()
        a, b = y.cpu().numpy(), y_ref.cpu().numpy()
        assert np.isfinite(b).all()
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32)), \
            f"call {call}: max diff {np.abs(a.astype(np.float64) - b).max()}"
    assert q.qmv_check() == 0


def test_moe_ffn_static_rejects_scratch_beyond_its_size():
    q.build()
    A = 0x10000
    inter = 32768
    n_sel = 8                                     # 8 * 32768 floats > the 131072-float array
    assert n_sel * inter > 8 * 16384
    rc = q.lib().moe_ffn_static(Q4_K, A, A, inter * 8 * 144, Q4_K, A, 1024 * 128 * 144, 16, A, A,
                                n_sel, 1024, inter, A, A, None)
    assert rc == -3                               # QMV_ERR_SHAPE, before anything is enqueued
