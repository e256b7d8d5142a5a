#!/usr/bin/env python
"""Benchmark of the quantized decode-step matvec on B200.

Headline step: the full decode-step matvec sweep of a 16-layer dense stack
(hidden 2048, intermediate 8192, 32 query / 8 KV heads of head_dim 64), all
weights Q8_0, one token: per layer the fused QKV 3072x2048, O 2048x2048, fused
gate/up 16384x2048 and down 2048x8192 matvecs -- 64 matvecs, 1.034 GB of
weights per step (larger than the 126 MB L2, so no flush is needed) -- run in
decode order (each matvec reads its x only after the previous one is complete,
as its input would be the previous output in a model): 64 library calls with
programmatic dependent launch (each launch may copy its weights while the
previous one finishes; --no-pdl turns it off), or with --mode chain one
qmv_chain call (the same launches, each also moving the next matvec's
weights into L2 once its own copies are issued).  The
step is captured once as a CUDA graph of the library's C-ABI calls and
replayed.
Metric: weight bytes streamed per second (GB/s), with the fraction of the
measured HBM peak.  The other workloads (Q8_0 1024^2, Q4_K fused QKV, Q6_K
vocab projection at 1 and 4 tokens, the MoE FFN step, the sweep at 2/4/8
tokens, and the sweep as independent grouped launches -- an upper bound for
matvecs that need no ordering) are measured in the same run and reported
under "per_config".

  python bench.py [--gpus N --steps K --warmup W]      # our CUDA path
  python bench.py --impl reference ...                   # the oracle on host cores
  python bench.py --profile-case q8_0|q4_k|q6_k          # one large matvec, for ncu

Multi-GPU: replicas only (the sweep does not shard across GPUs in this build):
each rank runs the same step on its own GPU, timed on the device, max over
ranks; value = all ranks' bytes / that time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from quantized_decode_superblocks_b200 import synth  # noqa: E402

Q8_0, Q4_K, Q6_K = synth.Q8_0, synth.Q4_K, synth.Q6_K
L2_BYTES = 126 * 1024 * 1024
METRIC = "quantized matvec µs and weight GB/s as % of B200 HBM peak (batch 1)"
WORKLOAD = ("16-layer Q8_0 decode-step matvec sweep, batch 1: per layer fused QKV 3072x2048, "
            "O 2048x2048, fused gate/up 16384x2048, down 2048x8192")


def bpw(fmt):
    return synth.BLOCK_BYTES[fmt] / synth.BLOCK_WEIGHTS[fmt]


def algo_bytes(fmt, rows, cols, n_tok):
    """Algorithmic bytes of one matvec: packed weights + x read + y written."""
    return synth.matrix_bytes(fmt, rows, cols) + 4 * n_tok * (cols + rows)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "quantized_decode_superblocks_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.endswith((".cu", ".cuh")):
            with open(os.path.join(csrc, name), "rb") as f:
                h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def step_config(n_tok):
    """The workload of a bench line, the same for both arms."""
    weight_bytes = sum(synth.matrix_bytes(Q8_0, rows, cols) for (_, _, _, rows, cols) in sweep_layers())
    return {"workload": WORKLOAD, "n_tok": n_tok, "layers": synth.CFG4_LAYERS,
            "weight_bytes_per_step": weight_bytes,
            "l2": "inputs larger than L2 (1.03 GB of weights per step, L2 126 MB)"}


def sweep_layers():
    return [(l, m, name, rows, cols) for l in range(synth.CFG4_LAYERS)
            for m, (name, rows, cols) in enumerate(synth.workload_cfg4_layer())]


# ------------------------------------------------------------------ clocks --

class ClockSampler:
    """nvidia-smi samples of this GPU's clocks and throttle reasons."""
    FIELDS = ("pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, props):
        b = getattr(props, "pci_bus_id", "")
        if not isinstance(b, str):
            try:
                b = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            except (AttributeError, TypeError, ValueError):
                b = ""
        self.bus = b.lower()
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader",
                                          "-lms", "200"], stdout=open(self.path, "w"),
                                         stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) < 9:
                        continue
                    bus = parts[0].lower()
                    if self.bus and not (bus.endswith(self.bus[-12:]) or self.bus.endswith(bus[-12:])):
                        continue
                    rows.append(parts)
            os.unlink(self.path)
        except OSError:
            pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}

        def num(v):
            try:
                return float(v.split()[0])
            except (ValueError, IndexError):
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------- device helpers --

class Dist:
    """Ranks of a torchrun launch: NCCL on GPUs (gloo for host-only tests).
    Only the timing is exchanged (barriers and a max over ranks): the sweep runs
    as an independent replica on every GPU."""

    def __init__(self, n_gpus):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        self.device = "cuda"
        if n_gpus > 1 and self.world != n_gpus:
            raise SystemExit(f"--gpus {n_gpus} needs torchrun with {n_gpus} ranks (WORLD_SIZE={self.world})")

    def init(self, torch, backend="nccl"):
        if backend == "nccl":
            torch.cuda.set_device(self.local)
        else:
            self.device = "cpu"
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
            self.pg = dist

    def barrier(self, torch):
        if self.pg is not None:
            if self.device == "cuda":
                self.pg.barrier(device_ids=[self.local])
            else:
                self.pg.barrier()

    def max(self, torch, v):
        if self.pg is None:
            return v
        t = torch.tensor([v], dtype=torch.float64, device=self.device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg is not None:
            self.pg.destroy_process_group()


def aggregate_gbs(bytes_per_step, world, steps, max_sec):
    """Whole-job throughput: every rank streams bytes_per_step per step; the job
    takes the slowest rank's time."""
    return bytes_per_step * world * steps / max_sec / 1e9


def time_graph(torch, graph, reps, stream):
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        start.record(stream)
        for _ in range(reps):
            graph.replay()
        end.record(stream)
    end.synchronize()
    return start.elapsed_time(end) / 1e3   # seconds


def capture(torch, fn, stream):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        fn()                        # warm: plans, attributes, lazy module loading
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=stream):
            fn()
    torch.cuda.synchronize()
    return g


# ----------------------------------------------------------- the sweep step --

class Sweep:
    """Device-resident weights / activations of the 16-layer Q8_0 sweep."""

    def __init__(self, torch, q, n_tok, host_cache):
        self.q, self.torch, self.n_tok = q, torch, n_tok
        self.mats = []
        x_off = y_off = 0
        for (l, m, name, rows, cols) in sweep_layers():
            key = (l, m)
            if key not in host_cache:
                host_cache[key] = synth.gen_blocks(Q8_0, rows, cols, synth.CFG4_SEED, 16 * l + m)
            self.mats.append(dict(rows=rows, cols=cols, W=torch.from_numpy(host_cache[key]).cuda(),
                                  x_off=x_off, y_off=y_off))
            x_off += n_tok * cols
            y_off += n_tok * rows
        xs = np.concatenate([synth.gen_x(n_tok, mm["cols"], synth.CFG4_SEED, 5000 + i).reshape(-1)
                             for i, mm in enumerate(self.mats)])
        self.x_host = torch.from_numpy(xs).pin_memory()
        self.x = self.x_host.cuda()
        self.y = torch.empty(y_off, device="cuda")
        self.y_host = torch.empty(y_off, dtype=torch.float32).pin_memory()
        self.weight_bytes = sum(synth.matrix_bytes(Q8_0, mm["rows"], mm["cols"]) for mm in self.mats)
        self.algo = sum(algo_bytes(Q8_0, mm["rows"], mm["cols"], n_tok) for mm in self.mats)
        self.tasks = q.make_tasks([(mm["W"], mm["rows"], mm["cols"], self.x.data_ptr() + 4 * mm["x_off"],
                                    self.y.data_ptr() + 4 * mm["y_off"]) for mm in self.mats])
        self.mode = "launches"
        self.launches = len(self.mats)

    def set_mode(self, mode):
        """'launches': one library call per matvec, in order; 'chain': the
        whole step as in-order chained calls (one token); 'grouped': the
        matvecs as independent grouped launches."""
        if mode == "chain" and self.n_tok != 1:
            raise ValueError("the chained step is one-token")
        self.mode = mode
        self.launches = {"launches": len(self.mats), "chain": len(self.mats),
                         "grouped": None}[mode]

    def launch(self, i, stream=None):
        mm = self.mats[i]
        x = self.x.data_ptr() + 4 * mm["x_off"]
        y = self.y.data_ptr() + 4 * mm["y_off"]
        if self.n_tok == 1:
            self.q.qmv_f32(Q8_0, mm["W"], mm["rows"], mm["cols"], x, y, stream)
        else:
            self.q.qmv_batched(Q8_0, mm["W"], mm["rows"], mm["cols"], x, y, self.n_tok, stream)

    def step(self, stream=None):
        if self.mode == "chain":
            self.q.qmv_chain(Q8_0, self.tasks, stream)
        elif self.mode == "grouped":
            self.q.qmv_multi(Q8_0, self.n_tok, self.tasks, stream)
        else:
            for i in range(len(self.mats)):
                self.launch(i, stream)


KERNEL_NAMES = {1: "warp-ring kernel", 2: "general pipeline kernel", 3: "tensor-core kernel",
                4: "streaming kernel"}


def per_kind_durations(torch, q, sweep, stream, reps=20):
    """Average duration of each projection type's launch as it runs in the
    step: a CUDA graph of that type's 16 launches (in layer order, same launch
    attributes), replayed and timed with CUDA events on the launch stream.
    Also returns which library kernel serves each type."""
    out, kernels = {}, {}
    layers = sweep_layers()
    for kind in dict.fromkeys(name for (_, _, name, _, _) in layers):
        idx = [i for i, (_, _, name, _, _) in enumerate(layers) if name == kind]
        g = capture(torch, lambda: [sweep.launch(i, stream) for i in idx], stream)
        kernels[kind] = KERNEL_NAMES.get(q.qmv_debug_last_kernel(), "?")
        time_graph(torch, g, 3, stream)
        out[kind] = (time_graph(torch, g, reps, stream) / (reps * len(idx)), len(idx))
        del g
    return out, kernels


# --------------------------------------------------------- per-config runs --

def rotating_pool(torch, fmt, rows, cols, seed, min_total):
    host = synth.gen_blocks(fmt, rows, cols, seed, 0)
    base = torch.from_numpy(host).cuda()
    copies = max(1, -(-min_total // host.nbytes))
    return [base] + [base.clone() for _ in range(copies - 1)]


POOL_L2_MULTIPLE = 4      # rotating weight pools hold at least this many L2s of data


def single_launch_us(torch, q, stream, fn, n, reps=30):
    """Median device time of ONE call fn(i) with programmatic dependent launch
    off: each call is bracketed by its own CUDA events on the launch stream,
    behind a ~20 µs sleep kernel so the host has queued both events and the
    call before the GPU reaches them (the events then time the GPU's work for
    that call alone, launch gap included).  fn(i) uses weight copy i % n."""
    pdl = q.qmv_get_pdl()
    q.qmv_set_pdl(0)
    out = []
    try:
        with torch.cuda.stream(stream):
            for i in range(reps + 3):
                ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                torch.cuda._sleep(40000)
                ev0.record(stream)
                fn(i % n)
                ev1.record(stream)
                ev1.synchronize()
                if i >= 3:
                    out.append(ev0.elapsed_time(ev1) * 1e3)
    finally:
        q.qmv_set_pdl(pdl)
    return statistics.median(out)


def measure_matvec(torch, q, stream, fmt, rows, cols, n_tok, seed, reps=200, argmax=False):
    """µs per matvec over a pool of weight copies of at least 4x L2: (a) a
    replayed graph of back-to-back launches with programmatic dependent launch
    (each launch's prologue and first weight copies overlap the previous
    launch: throughput of a stream of such matvecs), and (b) one launch alone,
    PDL off, event-timed (its latency).  argmax: the projection followed by
    the greedy argmax (qmv_argmax)."""
    pool = rotating_pool(torch, fmt, rows, cols, seed, POOL_L2_MULTIPLE * L2_BYTES)
    x = torch.from_numpy(synth.gen_x(n_tok, cols, seed, 1)).cuda()
    y = torch.empty((n_tok, rows), device="cuda")
    idx = torch.empty(n_tok, dtype=torch.int32, device="cuda")
    per_graph = len(pool) if len(pool) >= 64 else len(pool) * (64 // len(pool))

    def one(i):
        W = pool[i % len(pool)]
        if argmax:
            q.qmv_argmax(fmt, W, rows, cols, x, y, n_tok, idx)
        elif n_tok == 1:
            q.qmv_f32(fmt, W, rows, cols, x, y)
        else:
            q.qmv_batched(fmt, W, rows, cols, x, y, n_tok)

    def body():
        for i in range(per_graph):
            one(i)
    g = capture(torch, body, stream)
    time_graph(torch, g, 3, stream)
    n_rep = max(2, reps // per_graph)
    sec = time_graph(torch, g, n_rep, stream) / (n_rep * per_graph)
    del g
    wb = synth.matrix_bytes(fmt, rows, cols)
    us1 = single_launch_us(torch, q, stream, one, len(pool))
    return {"fmt": synth.FORMAT_NAMES[fmt], "rows": rows, "cols": cols, "n_tok": n_tok,
            "us": sec * 1e6, "weight_gbs": wb / sec / 1e9, "copies": len(pool),
            "pool_bytes": wb * len(pool),
            "timing": "graph of back-to-back launches, programmatic dependent launch on (pipelined)",
            "us_single_launch": round(us1, 3), "weight_gbs_single_launch": round(wb / us1 / 1e3, 1),
            "single_launch_timing": "one launch, PDL off, CUDA events around it"}


def measure_moe(torch, q, stream, reps=200, separate=False):
    """The MoE FFN step of the 32-expert workload: moe_ffn_routed (router and
    both products in one launch), or with separate=True moe_route followed by
    moe_ffn (three launches)."""
    w = synth.workload_cfg3()
    E, hidden, inter, seed = w["n_expert"], w["hidden"], w["inter"], w["seed"]
    gus = synth.matrix_bytes(Q4_K, inter, hidden)
    ds = synth.matrix_bytes(Q4_K, hidden, inter)
    host = [synth.gen_blocks(Q4_K, inter * E, hidden, seed, 1), synth.gen_blocks(Q4_K, inter * E, hidden, seed, 2),
            synth.gen_blocks(Q4_K, hidden * E, inter, seed, 3)]
    base = [torch.from_numpy(h).cuda() for h in host]
    touched = 4 * (2 * gus + ds)
    # each step touches 24.8 MB of the selected experts: enough copies that the
    # steps of one graph replay cycle through at least 4x L2 of weights
    n_copies = -(-POOL_L2_MULTIPLE * L2_BYTES // touched)
    sets = [base] + [[t.clone() for t in base] for _ in range(n_copies - 1)]
    logits, bias = synth.gen_router(E, seed, 5)
    lg, bs = torch.from_numpy(logits).cuda(), torch.from_numpy(bias).cuda()
    x = torch.from_numpy(synth.gen_x(1, hidden, seed, 4)[0]).cuda()
    ids = torch.empty(4, dtype=torch.int32, device="cuda")
    g = torch.empty(4, device="cuda")
    h = torch.empty((4, inter), device="cuda")
    y = torch.empty(hidden, device="cuda")
    ws = torch.zeros(q.MOE_WS_BYTES // 8, dtype=torch.int64, device="cuda")
    per_graph = 2 * n_copies

    def one(i):
        G, U, D = sets[i % n_copies]
        if separate:
            q.moe_route(lg, bs, E, 4, ids, g)
            q.moe_ffn(Q4_K, G, U, gus, Q4_K, D, ds, E, ids, g, 4, hidden, inter, x, h, y)
        else:
            q.moe_ffn_routed(lg, bs, E, 4, Q4_K, G, U, gus, Q4_K, D, ds, hidden, inter, x, ids, g, h, y, ws)

    def body():
        for i in range(per_graph):
            one(i)
    gr = capture(torch, body, stream)
    time_graph(torch, gr, 3, stream)
    n_rep = max(2, reps // per_graph)
    sec = time_graph(torch, gr, n_rep, stream) / (n_rep * per_graph)
    del gr
    us1 = single_launch_us(torch, q, stream, one, n_copies)
    return {"workload": "MoE FFN step: route top-4 of 32 + Q4_K gate/up 1792x2048 + down 2048x1792",
            "calls": "moe_route + moe_ffn" if separate else "moe_ffn_routed",
            "us": sec * 1e6, "weight_gbs": touched / sec / 1e9,
            "weight_bytes_touched": touched, "copies": n_copies,
            "timing": "graph of back-to-back steps, programmatic dependent launch on (pipelined)",
            "us_single_launch": round(us1, 3), "weight_gbs_single_launch": round(touched / us1 / 1e3, 1),
            "single_launch_timing": "one step alone, PDL off, CUDA events around it"}


def measure_lfm_mix(torch, q, stream, reps=10):
    """One decode token of the LFM2.5-style 24-layer mix (synth.workload_lfm_mix):
    per layer the attention (fused QK, V, O) or short-convolution (in / out
    projection) matvecs, then the routed MoE FFN step (moe_ffn_routed, its own
    router logits per layer), and finally the vocabulary projection with greedy
    argmax -- 79 library calls in decode order, captured as one CUDA graph.
    Every layer has its own weights on the device (4.9 GB in all, each layer's
    a block-rotated copy of one generated set, so no two layers share data);
    a token streams about 1 GB of them.  Activations chain from call to call
    (each call reads the previous output) without norms or the convolution
    and attention arithmetic, which are not matvecs: a bandwidth workload, not
    a forward pass."""
    w = synth.workload_lfm_mix()
    seed, L, mo = w["seed"], w["layers"], w["moe"]
    E, hidden, inter, top_k = mo["n_expert"], mo["hidden"], mo["inter"], mo["top_k"]

    def rotated(host, fmt, layer):
        t = torch.from_numpy(host).cuda()
        nb = host.size // synth.BLOCK_BYTES[fmt]
        return torch.roll(t, shifts=int((layer * 7919) % nb) * synth.BLOCK_BYTES[fmt]) if layer else t

    base = {}
    for name, fmt, rows, cols in w["attention"] + w["conv"]:
        base[name] = (fmt, rows, cols, synth.gen_blocks(fmt, rows, cols, seed, len(base) + 1))
    gus, ds = synth.matrix_bytes(Q4_K, inter, hidden), synth.matrix_bytes(Q4_K, hidden, inter)
    ex_host = [synth.gen_blocks(Q4_K, inter * E, hidden, seed, 10), synth.gen_blocks(Q4_K, inter * E, hidden, seed, 11),
               synth.gen_blocks(Q4_K, hidden * E, inter, seed, 12)]
    vf, vrows, vcols = w["vocab"]
    vocab = torch.from_numpy(synth.gen_blocks(vf, vrows, vcols, seed, 13)).cuda()
    layers = []
    touched = synth.matrix_bytes(vf, vrows, vcols)
    for l in range(L):
        kind = "attention" if synth.lfm_attention_layer(l) else "conv"
        mats = [(base[n][0], base[n][1], base[n][2], rotated(base[n][3], base[n][0], l)) for n, *_ in w[kind]]
        experts = [rotated(h, Q4_K, l) for h in ex_host]
        logits, bias = synth.gen_router(E, seed, 100 + l)
        layers.append((kind, mats, experts, torch.from_numpy(logits).cuda(), torch.from_numpy(bias).cuda()))
        touched += sum(synth.matrix_bytes(f, r, c) for f, r, c, _ in mats) + top_k * (2 * gus + ds)
    h = torch.from_numpy(synth.gen_x(1, hidden, seed, 20)[0]).cuda()
    h2 = torch.empty(hidden, device="cuda")
    y_big = torch.empty(3 * hidden, device="cuda")
    y_v = torch.empty(512, device="cuda")
    ids = torch.empty(top_k, dtype=torch.int32, device="cuda")
    g = torch.empty(top_k, device="cuda")
    hs = torch.empty((top_k, inter), device="cuda")
    ws = torch.zeros(q.MOE_WS_BYTES // 8, dtype=torch.int64, device="cuda")
    vlog = torch.empty(vrows, device="cuda")
    idx = torch.empty(1, dtype=torch.int32, device="cuda")
    n_calls = 0

    def token():
        nonlocal n_calls
        n_calls = 0
        for kind, mats, (G, U, D), lg, bs in layers:
            if kind == "attention":
                (fq, rq, cq, Wq), (fv, rv, cv, Wv), (fo, ro, co, Wo) = mats
                q.qmv_f32(fq, Wq, rq, cq, h, y_big)
                q.qmv_f32(fv, Wv, rv, cv, h, y_v)
                q.qmv_f32(fo, Wo, ro, co, y_big, h2)           # stand-in for the attention output
                n_calls += 3
            else:
                (fi, ri, ci, Wi), (fo, ro, co, Wo) = mats
                q.qmv_f32(fi, Wi, ri, ci, h, y_big)
                q.qmv_f32(fo, Wo, ro, co, y_big, h2)           # stand-in for the gated convolution output
                n_calls += 2
            q.moe_ffn_routed(lg, bs, E, top_k, Q4_K, G, U, gus, Q4_K, D, ds, hidden, inter, h2, ids, g, hs, h, ws)
            n_calls += 1
        q.qmv_argmax(vf, vocab, vrows, vcols, h, vlog, 1, idx)
        n_calls += 1

    gr = capture(torch, token, stream)
    time_graph(torch, gr, 3, stream)
    sec = time_graph(torch, gr, reps, stream) / reps
    del gr
    assert q.qmv_check(stream) == 0
    return {"workload": "LFM2.5-style decode token: 24 layers (6 attention: QK 2560x2048 Q4_K, V 512x2048 Q6_K, "
                        "O 2048x2048 Q4_K; 18 short convolution: in 6144x2048, out 2048x2048 Q4_K), a top-4-of-32 "
                        "Q4_K MoE FFN (1792) per layer, Q6_K vocabulary 128000x2048 with greedy argmax",
            "calls": f"{n_calls} library calls per token (qmv_f32, moe_ffn_routed, qmv_argmax) in one CUDA graph",
            "us": sec * 1e6, "tokens_per_s": round(1.0 / sec, 1), "weight_gbs": touched / sec / 1e9,
            "weight_bytes_per_token": touched,
            "timing": "graph of one token's calls, replayed; CUDA events; weights of all 24 layers resident "
                      "(no L2 reuse across layers)"}


# ----------------------------------------------------------- reference arm --

def cpu_info():
    """CPU model, physical cores and logical CPUs of this host (lscpu)."""
    info = {"model": None, "physical_cores": None, "logical_cpus": os.cpu_count()}
    try:
        out = subprocess.run(["lscpu"], capture_output=True, text=True, timeout=10).stdout
        kv = {}
        for line in out.splitlines():
            if ":" in line:
                k, v = line.split(":", 1)
                kv[k.strip()] = v.strip()
        info["model"] = kv.get("Model name")
        cps, sockets = kv.get("Core(s) per socket"), kv.get("Socket(s)")
        if cps and sockets and cps.isdigit() and sockets.isdigit():
            info["physical_cores"] = int(cps) * int(sockets)
    except (OSError, subprocess.SubprocessError):
        pass
    return info


def oracle_baseline(seconds_single, seconds_all, cache):
    """The oracle timed on this host's cores over a bounded sample of the sweep
    (layer 0's four Q8_0 matvecs): single-threaded and with OpenMP over rows on
    every logical CPU, each the median GB/s of 5 timed passes."""
    import oracle
    info = cpu_info()
    out = {}
    for label, threads, secs in (("single_thread", 1, seconds_single),
                                 ("all_cores", os.cpu_count() or 1, seconds_all)):
        rate, used, sample = oracle_rate(secs, cache, threads)
        out[label] = {"value": round(rate, 3), "cores": used, "sample": sample}
    return {"value": out["all_cores"]["value"], "unit": "GB/s", "cores": out["all_cores"]["cores"],
            "kind": "oracle", "sample": out["all_cores"]["sample"],
            "single_thread": {"value": out["single_thread"]["value"], "unit": "GB/s", "cores": 1,
                              "sample": out["single_thread"]["sample"]},
            "cpu_model": info["model"], "physical_cores": info["physical_cores"],
            "logical_cpus": info["logical_cpus"],
            "method": "oracle (plain C, f64 accumulation, OpenMP over rows), median of 5 timed passes"}


def oracle_rate(seconds, cache, threads=None):
    """The oracle on the host cores over a bounded sample of the sweep: GB/s of
    weight bytes (median of 5 passes, each about seconds / 5), the threads it
    used, and the sample description."""
    import oracle
    threads = threads or os.cpu_count() or 1
    mats = [(l, m, name, rows, cols) for (l, m, name, rows, cols) in sweep_layers() if l == 0]
    data = []
    for (l, m, name, rows, cols) in mats:
        key = (l, m)
        if key not in cache:
            cache[key] = synth.gen_blocks(Q8_0, rows, cols, synth.CFG4_SEED, 16 * l + m)
        data.append((cache[key], rows, cols, synth.gen_x(1, cols, synth.CFG4_SEED, 5000 + m)))
    rates, total_t, total_passes = [], 0.0, 0
    for _ in range(5):
        done_bytes, t0, passes = 0, time.perf_counter(), 0
        while True:
            for W, rows, cols, x in data:
                oracle.qmv(Q8_0, W, rows, cols, x, nthreads=threads)
                done_bytes += W.nbytes
            passes += 1
            if time.perf_counter() - t0 >= seconds / 5:
                break
        dt = time.perf_counter() - t0
        rates.append(done_bytes / dt / 1e9)
        total_t += dt
        total_passes += passes
    return (statistics.median(rates), threads,
            f"{total_passes} passes over layer 0's four Q8_0 matvecs ({total_t:.1f} s, {threads} threads)")


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    cache = {}
    # calibrate, then size each step's sample so warm-up + timed steps take ~60 s
    rate, threads, _ = oracle_rate(1.0, cache)
    per_step_bytes = max(1, int(rate * 1e9 * 60.0 / max(1, args.steps + args.warmup)))
    W0, rows0, cols0 = cache[(0, 2)], 16384, 2048
    row_bytes = W0.nbytes // rows0
    n_rows = max(1, min(rows0, per_step_bytes // row_bytes))
    x = synth.gen_x(1, cols0, synth.CFG4_SEED, 5002)
    sub = W0[: n_rows * row_bytes]
    for _ in range(args.warmup):
        oracle.qmv(Q8_0, sub, n_rows, cols0, x, nthreads=threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.qmv(Q8_0, sub, n_rows, cols0, x, nthreads=threads)
    dt = time.perf_counter() - t0
    value = n_rows * row_bytes * args.steps / dt / 1e9
    sample = f"each step: {n_rows} rows of the 16384x2048 Q8_0 gate/up matvec ({n_rows * row_bytes} B)"
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "GB/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt / args.steps * 1e3, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": step_config(args.n_tok),
            "run": {"parallelism": "host cores (oracle)"},
            "cpu_baseline": {"value": round(value, 3), "unit": "GB/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 3), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------ profile case --

PROFILE_CASES = {
    # name: (fmt, rows, cols) -- one matvec, a few launches, < 1 GB on the device
    "q8_0": (Q8_0, 65536, 2048), "q4_k": (Q4_K, 131072, 2048), "q6_k": (Q6_K, 96000, 2048),
    "q8_0_down": (Q8_0, 16384, 8192), "q8_0_o": (Q8_0, 2048, 2048),
    "gate_up": (Q8_0, 16384, 2048), "down": (Q8_0, 2048, 8192), "qkv": (Q8_0, 3072, 2048),
    "cfg0": (Q8_0, 1024, 1024), "cfg1": (Q4_K, 3072, 2048), "cfg2": (Q6_K, 128000, 2048),
}


def run_profile_moe(args):
    """A few MoE FFN steps of the 32-expert workload, 198 MB of experts on the
    device: moe_ffn_routed (one launch), then moe_route + moe_ffn (three)."""
    import torch
    import quantized_decode_superblocks_b200 as q
    torch.cuda.set_device(0)
    w = synth.workload_cfg3()
    E, hidden, inter, seed = w["n_expert"], w["hidden"], w["inter"], w["seed"]
    gus, ds = synth.matrix_bytes(Q4_K, inter, hidden), synth.matrix_bytes(Q4_K, hidden, inter)
    G = torch.from_numpy(synth.gen_blocks(Q4_K, inter * E, hidden, seed, 1)).cuda()
    U = torch.from_numpy(synth.gen_blocks(Q4_K, inter * E, hidden, seed, 2)).cuda()
    D = torch.from_numpy(synth.gen_blocks(Q4_K, hidden * E, inter, seed, 3)).cuda()
    logits, bias = synth.gen_router(E, seed, 5)
    lg, bs = torch.from_numpy(logits).cuda(), torch.from_numpy(bias).cuda()
    x = torch.from_numpy(synth.gen_x(1, hidden, seed, 4)[0]).cuda()
    ids = torch.empty(4, dtype=torch.int32, device="cuda")
    g = torch.empty(4, device="cuda")
    h = torch.empty((4, inter), device="cuda")
    y = torch.empty(hidden, device="cuda")
    ws = torch.zeros(q.MOE_WS_BYTES // 8, dtype=torch.int64, device="cuda")
    for _ in range(max(1, args.steps)):
        q.moe_ffn_routed(lg, bs, E, 4, Q4_K, G, U, gus, Q4_K, D, ds, hidden, inter, x, ids, g, h, y, ws)
    for _ in range(max(1, args.steps)):
        q.moe_route(lg, bs, E, 4, ids, g)
        q.moe_ffn(Q4_K, G, U, gus, Q4_K, D, ds, E, ids, g, 4, hidden, inter, x, h, y)
    torch.cuda.synchronize()
    assert q.qmv_check() == 0
    print(json.dumps({"profile_case": "moe", "weight_bytes_touched": 4 * (2 * gus + ds)}))
    return 0


def run_profile_case(args):
    """A few launches of one matvec -- the small case that ncu captures."""
    if args.profile_case == "moe":
        return run_profile_moe(args)
    import torch
    import quantized_decode_superblocks_b200 as q
    fmt, rows, cols = PROFILE_CASES[args.profile_case]
    torch.cuda.set_device(0)
    W = torch.from_numpy(synth.gen_blocks(fmt, rows, cols, 77, 0)).cuda()
    x = torch.from_numpy(synth.gen_x(args.n_tok, cols, 77, 1)).cuda()
    y = torch.empty((args.n_tok, rows), device="cuda")
    for _ in range(max(1, args.steps)):
        q.qmv_batched(fmt, W, rows, cols, x, y, args.n_tok)
    torch.cuda.synchronize()
    assert q.qmv_check() == 0
    print(json.dumps({"profile_case": args.profile_case, "rows": rows, "cols": cols, "n_tok": args.n_tok,
                      "weight_bytes": synth.matrix_bytes(fmt, rows, cols)}))
    return 0


# --------------------------------------------------------------------- main --

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--n-tok", type=int, default=1)
    ap.add_argument("--mode", choices=["launches", "chain"], default="launches",
                    help="how the step runs, in decode order either way: 'launches' = one library "
                         "call per matvec (default), 'chain' = one qmv_chain call (the same launches, "
                         "each moving the next matvec's weights into L2; one token)")
    ap.add_argument("--no-pdl", action="store_true",
                    help="launch without programmatic dependent launch (qmv_set_pdl(0))")
    ap.add_argument("--headline-only", action="store_true",
                    help="skip the per-config measurements and the CPU baseline")
    ap.add_argument("--profile-case", choices=sorted(PROFILE_CASES) + ["moe"])
    args = ap.parse_args()
    if args.warmup < 3 and not args.profile_case:
        raise SystemExit("--warmup must be at least 3")
    if args.impl == "reference":
        return run_reference(args)
    if args.profile_case:
        return run_profile_case(args)

    import torch
    import quantized_decode_superblocks_b200 as q
    dist = Dist(args.gpus)
    dist.init(torch)
    q.lib()                                  # fails loudly if the library is missing
    stream = torch.cuda.Stream()
    hbm_peak, peak_kind = peaks()
    props = torch.cuda.get_device_properties(torch.cuda.current_device())
    cache = {}

    mode = args.mode
    q.qmv_set_pdl(0 if args.no_pdl else 1)
    sweep = Sweep(torch, q, args.n_tok, cache)
    sweep.set_mode(mode)
    graph = capture(torch, lambda: sweep.step(), stream)
    assert q.qmv_check(stream) == 0

    per_config = {}
    with ClockSampler(props) as clk:
        # warm-up, then the timed steps (device time, barrier + sync on both sides)
        with torch.cuda.stream(stream):
            for _ in range(args.warmup):
                graph.replay()
        torch.cuda.synchronize()
        dist.barrier(torch)
        torch.cuda.synchronize()
        sec = time_graph(torch, graph, args.steps, stream)
        torch.cuda.synchronize()
        dist.barrier(torch)
        sec = dist.max(torch, sec)
        # the dominant kernel: every launch of the step, event-timed on its stream
        durs, kinds = per_kind_durations(torch, q, sweep, stream)
        # end to end: pinned x -> device, the step's library calls, y -> pinned host
        e2e_reps = max(3, min(200, args.steps // 5))
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        ev0.record(stream)
        with torch.cuda.stream(stream):
            for _ in range(e2e_reps):
                sweep.x.copy_(sweep.x_host, non_blocking=True)
                graph.replay()
                sweep.y_host.copy_(sweep.y, non_blocking=True)
        ev1.record(stream)
        ev1.synchronize()
        e2e_sec = dist.max(torch, ev0.elapsed_time(ev1) / 1e3 / e2e_reps)
        if not args.headline_only and dist.rank == 0:
            per_config["cfg0_q8_0_1024x1024"] = measure_matvec(torch, q, stream, Q8_0, 1024, 1024, 1, 0)
            per_config["cfg1_q4_k_fused_qkv_3072x2048"] = measure_matvec(torch, q, stream, Q4_K, 3072, 2048, 1, 1)
            for nt in (1, 4):
                per_config[f"cfg2_q6_k_vocab_128000x2048_ntok{nt}"] = measure_matvec(
                    torch, q, stream, Q6_K, 128000, 2048, nt, 2, reps=20)
            per_config["cfg2_q6_k_vocab_128000x2048_ntok1_greedy_argmax"] = measure_matvec(
                torch, q, stream, Q6_K, 128000, 2048, 1, 2, reps=20, argmax=True)
            per_config["cfg3_moe_ffn_step"] = measure_moe(torch, q, stream)
            per_config["cfg3_moe_route_then_ffn"] = measure_moe(torch, q, stream, separate=True)
            per_config["lfm2_5_style_mix_token"] = measure_lfm_mix(torch, q, stream)
            torch.cuda.empty_cache()
            for nt in (1, 2, 4, 8):
                sw = Sweep(torch, q, nt, cache)
                for md in (("launches", "chain", "grouped") if nt == 1 else ("launches", "grouped")):
                    if nt == args.n_tok and md == mode:
                        continue
                    sw.set_mode(md)
                    gr = capture(torch, lambda: sw.step(), stream)
                    reps = max(3, args.steps // 10)
                    s2 = time_graph(torch, gr, reps, stream) / reps
                    key = f"cfg4_sweep_ntok{nt}" + ("" if md == "launches" else f"_{md}")
                    per_config[key] = {"us": s2 * 1e6, "weight_gbs": sw.weight_bytes / s2 / 1e9,
                                       "launches": sw.launches, "mode": md,
                                       "order": "independent (grouped, no ordering)" if md == "grouped"
                                       else "decode order"}
                    del gr
                del sw
    clocks = clk.summary()
    assert q.qmv_check(stream) == 0

    value = aggregate_gbs(sweep.weight_bytes, dist.world, args.steps, sec)
    ms_per_step = sec / args.steps * 1e3
    # the dominant kernel: the projection type with the largest share of the
    # step's kernel time; achieved = its algorithmic bytes per launch / its
    # average event-timed duration
    shapes = {name: (rows, cols) for (_, _, name, rows, cols) in sweep_layers()}
    total_kernel_sec = sum(sec1 * n for sec1, n in durs.values())
    dom_name = max(durs, key=lambda k: durs[k][0] * durs[k][1])
    dom_launch_sec, dom_n = durs[dom_name]
    dom_share = dom_launch_sec * dom_n / total_kernel_sec
    shares = {k: round(v[0] * v[1] / total_kernel_sec, 4) for k, v in durs.items()}
    rows, cols = shapes[dom_name]
    dom_bytes = algo_bytes(Q8_0, rows, cols, args.n_tok)
    dom_kernel = f"Q8_0 {dom_name} matvec {rows}x{cols} ({kinds[dom_name]}), {dom_n} launches per step"
    achieved = dom_bytes / dom_launch_sec / 1e9
    traffic = None
    tpath = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if os.path.exists(tpath):
        with open(tpath) as f:
            t = json.load(f)
        if (t.get("source_hash") == source_hash() and t.get("n_tok") == args.n_tok
                and t.get("kernel") == dom_name):
            traffic = t.get("traffic_bytes_per_launch")
    cfg4_key = f"cfg4_sweep_ntok{args.n_tok}" + ("" if mode == "launches" else f"_{mode}")
    per_config[cfg4_key] = {"us": ms_per_step * 1e3, "weight_gbs": sweep.weight_bytes / (sec / args.steps) / 1e9,
                            "launches": sweep.launches, "mode": mode, "order": "decode order"}
    for v in per_config.values():
        if "weight_gbs" in v:
            v["frac_of_hbm_peak"] = round(v["weight_gbs"] / hbm_peak, 4)
            v["us"] = round(v["us"], 3)
            v["weight_gbs"] = round(v["weight_gbs"], 1)

    cpu = None
    if dist.rank == 0 and args.gpus == 1 and not args.headline_only:
        cpu = oracle_baseline(8.0, 8.0, cache)

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": step_config(args.n_tok),
        "run": {"launches_per_step": sweep.launches,
                "timing": "CUDA graph of the step's C-ABI calls, replayed; CUDA events on the launch stream",
                "mode": mode,
                "pdl": not args.no_pdl,
                "order": "decode order: every matvec reads its x after the previous one has finished",
                "parallelism": f"replicas x{args.gpus}" if args.gpus > 1 else "single GPU"},
        "frac_of_hbm_peak": round(value / dist.world / hbm_peak, 4),
        "us_per_step": round(ms_per_step * 1e3, 2),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
                     "frac": round(achieved / hbm_peak, 4), "traffic": traffic,
                     "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured" else "fallback 6.65 TB/s",
                     "kernel": dom_kernel,
                     "algorithmic_bytes_per_launch": dom_bytes,
                     "launch_us": round(dom_launch_sec * 1e6, 3),
                     "share_of_step_kernel_time": round(dom_share, 4),
                     "kernel_time_shares": shares,
                     "step_kernel_gbs": round(sweep.algo / total_kernel_sec / 1e9, 1),
                     "timing": "each projection type's 16 launches as a replayed CUDA graph, CUDA events"},
        "e2e": {"value": round(sweep.weight_bytes * dist.world / e2e_sec / 1e9, 1), "unit": "GB/s",
                "h2d_bytes_per_step": int(sweep.x_host.numel() * 4),
                "d2h_bytes_per_step": int(sweep.y_host.numel() * 4)},
        "gpu_launches": sweep.launches * args.steps,
        "clocks": clocks,
        "cpu_baseline": cpu,
        "per_config": per_config,
    }
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    del graph
    dist.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
