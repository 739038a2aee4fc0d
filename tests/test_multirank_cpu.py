"""The bench's N>1 host logic with two gloo ranks on CPU: per-rank batches,
max-over-ranks timing, the whole-job weak-scaling value, and the reference arm
running on rank 0 only."""
import contextlib
import datetime
import io
import os
import socket

import numpy as np
import pytest


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from synth import WORKLOADS, make_routing
        import oracle as orc
        w = WORKLOADS["tiny"]
        seed = bench.rank_seed(w.seed, rank)
        ids = make_routing(w, seed=seed, T=1024)
        st = orc.coact(ids, w.E)
        ms = [3.0, 5.0, 4.0][rank]
        got = bench.reduce_max(ms, dist, torch.device("cpu"))
        tot = torch.tensor([float(st["coact"][0].trace())])
        dist.all_reduce(tot)
        q.put((rank, seed, got, int(ids.sum()), float(tot.item())))
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_two_gloo_ranks(world):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    seeds = [r[1] for r in res]
    assert len(set(seeds)) == world                       # independent batches
    assert len(set(r[3] for r in res)) == world
    assert all(r[2] == 5.0 for r in res)                  # max over ranks
    assert all(r[4] == world * 1024 * 2 for r in res)     # sum of traces = ranks * T * k


def test_weak_value_formula():
    import bench
    assert bench.weak_value(4, 2e9, 10.0) == pytest.approx(4 * 2e9 / 0.01 / 1e9)
    assert bench.reduce_max(7.5, None, None) == 7.5


def test_reference_arm_rank_nonzero_does_nothing(monkeypatch):
    import bench
    from synth import WORKLOADS
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class A:
        steps, warmup, gpus, placement, no_shuffle, balanced_shuffle = 1, 0, 2, "correlated", False, False
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(A(), WORKLOADS["tiny"])
    assert buf.getvalue() == ""


def test_reference_arm_prints_contract_line(monkeypatch):
    import json
    import bench
    from synth import WORKLOADS
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")

    class A:
        steps, warmup, gpus, placement, no_shuffle, balanced_shuffle = 1, 0, 1, "correlated", False, False
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(A(), WORKLOADS["tiny"])
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["higher_is_better"] is True
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["config"]["workload"] == "tiny"


def test_measured_peaks_file(monkeypatch, tmp_path):
    """The roofline denominators come from MEASURED_PEAKS.json when it holds
    them (plain numbers or {"value": ...}), else the fallbacks."""
    import json
    import bench
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.peaks() == (bench.FALLBACK_HBM_GBS, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6559.4, "bf16_tflops": {"value": 1585.0}}))
    assert bench.peaks() == (6559.4, "measured")
    assert bench.tensor_peak() == (1585.0, "measured")
    (tmp_path / "MEASURED_PEAKS.json").write_text("{not json")
    assert bench.peaks() == (bench.FALLBACK_HBM_GBS, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": None}))
    assert bench.tensor_peak() == (1590.0, "fallback") and bench.peaks()[1] == "fallback"
