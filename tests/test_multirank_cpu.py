"""Host logic of the multi-GPU benchmark path, run as two gloo ranks on the
CPU: each rank decodes its own request (its own inputs), the time is the
maximum over ranks, and the whole-job value counts every rank's beam-head
steps.  The decode step itself has no exchange between ranks, so nothing
else crosses ranks."""
import importlib.util
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        bench = _bench()
        import synth
        wl = bench.rank_workload(synth.workload("tiny"), rank)
        steps = synth.draw_decode(wl)
        # A per-rank "device time": rank 1 is the slow one.
        local_ms = 2.0 + 3.0 * rank
        mx = bench.max_over_ranks(local_ms, "cpu")
        dist.barrier()
        val = bench.whole_job_value(wl.units, world, mx)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"max": mx, "value": val, "seed": wl.seed_id,
                       "q0": steps[0]["q"].float().flatten()[:8].tolist()}, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_time_and_inputs(tmp_path):
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    r0 = json.load(open(tmp_path / "rank0.json"))
    r1 = json.load(open(tmp_path / "rank1.json"))
    assert r0["max"] == r1["max"] == 5.0          # the slowest rank sets the time
    import synth
    units = synth.workload("tiny").units
    assert r0["value"] == r1["value"] == pytest.approx(units * 2 / 5e-3)
    assert r0["seed"] != r1["seed"]               # every rank has its own request
    assert r0["q0"] != r1["q0"]


def test_single_process_needs_no_process_group():
    bench = _bench()
    assert bench.max_over_ranks(3.5, "cpu") == 3.5
    assert bench.whole_job_value(100, 1, 2.0) == pytest.approx(5e4)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    bench = _bench()
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    args = type("A", (), {"workload": "tiny", "steps": 1, "warmup": 0})()
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(args)
    assert buf.getvalue() == ""
