"""Host-side logic of bench.py (no GPU): the multi-rank timing exchange over
gloo with two ranks, the whole-job throughput formula, the clock-sample
summary, and the reference arm's rank handling."""
from __future__ import annotations

import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    d = bench.Dist(world)
    d.init(torch, backend="gloo")
    d.barrier(torch)
    local = 0.010 * (rank + 1)            # rank 1 is the slow one
    m = d.max(torch, local)
    out[rank] = (m, bench.aggregate_gbs(1e9, d.world, 10, m))
    d.barrier(torch)
    d.close()


def test_two_rank_max_over_ranks_gloo():
    port = _free_port()
    with mp.Manager() as man:
        out = man.dict()
        mp.start_processes(_rank_main, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
        res = dict(out)
    assert set(res) == {0, 1}
    for m, gbs in res.values():
        assert m == pytest.approx(0.020)
        # 2 ranks x 10 steps x 1 GB in the slowest rank's 20 ms
        assert gbs == pytest.approx(2 * 10 * 1.0 / 0.020)


def test_single_rank_needs_no_process_group(monkeypatch):
    monkeypatch.setenv("WORLD_SIZE", "1")
    d = bench.Dist(1)
    d.init(torch, backend="gloo")
    assert d.pg is None and d.max(torch, 1.5) == 1.5


def test_gpus_without_torchrun_is_an_error(monkeypatch):
    monkeypatch.setenv("WORLD_SIZE", "1")
    with pytest.raises(SystemExit):
        bench.Dist(2)


def test_clock_summary(tmp_path):
    class P:
        pci_bus_id = "00000000:1B:00.0"
    c = bench.ClockSampler(P())
    c.path = str(tmp_path / "c.csv")
    with open(c.path, "w") as f:
        f.write("00000000:1B:00.0, 1900 MHz, 1965 MHz, 800.0 W, 0x0, Not Active, Not Active, Not Active, Not Active\n")
        f.write("00000000:1B:00.0, 1800 MHz, 1965 MHz, 990.0 W, 0x4, Not Active, Not Active, Not Active, Active\n")
        f.write("00000000:2A:00.0, 500 MHz, 1965 MHz, 90.0 W, 0x0, Active, Not Active, Not Active, Not Active\n")
    s = c.summary()
    assert s["samples"] == 2 and s["sm_mhz"] == 1850 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"]


def test_reference_arm_other_ranks_exit_quietly(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")

    class A:
        steps, warmup, gpus = 10, 3, 2
    assert bench.run_reference(A()) == 0
    assert capsys.readouterr().out == ""
