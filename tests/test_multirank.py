"""Host logic of the multi-GPU bench on CPU: two gloo ranks (no GPU, no collective on the data path)."""

import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, ws, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(ws), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    import bench
    w, r, _ = bench.setup_dist()
    assert (w, r) == (ws, rank)
    cfg = bench.rank_config(bench.CFG, w, r)
    # each rank's step time differs; every rank must see the slowest one
    mx = bench.max_over_ranks(1.0 + rank, w)
    bench.barrier(w)
    value = bench.job_throughput(w, cfg.B * cfg.n, mx)
    out[rank] = (cfg.seed, mx, value)
    import torch.distributed as dist
    dist.destroy_process_group()


def test_two_ranks_take_the_max_and_use_their_own_seeds():
    ws = 2
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(ws, _free_port(), out), nprocs=ws, join=True)
    seeds = {out[r][0] for r in range(ws)}
    assert len(seeds) == ws                       # distinct batches per rank (weak scaling)
    assert all(out[r][1] == 2.0 for r in range(ws))   # max over ranks
    import bench
    T = bench.CFG.B * bench.CFG.n
    assert all(abs(out[r][2] - ws * T / 2e-3) < 1e-6 for r in range(ws))


def test_reference_arm_runs_on_rank_zero_only(capsys):
    import argparse
    import bench
    bench.run_reference(argparse.Namespace(steps=1, warmup=0), 2, 1)   # rank 1: no work, no output
    assert capsys.readouterr().out == ""


def test_reference_arm_prints_the_contract_line(capsys):
    import argparse
    import json
    import bench
    bench.run_reference(argparse.Namespace(steps=1, warmup=0), 1, 0)
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["higher_is_better"] is True and d["value"] > 0 and d["steps"] == 1
    assert d["config"]["workload"] == bench.CFG.name
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_gpus_flag_relaunches_one_rank_per_gpu(monkeypatch):
    """bench.py --gpus N started without a launcher runs itself as N ranks; under a launcher the
    world size must match N."""
    import sys
    import bench
    calls = []
    monkeypatch.setattr(bench, "relaunch_ranks", lambda n: calls.append(n) or 0)
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    monkeypatch.setattr(sys, "argv", ["bench.py", "--gpus", "2", "--steps", "3"])
    with pytest.raises(SystemExit) as e:
        bench.main()
    assert e.value.code == 0 and calls == [2]
    monkeypatch.setenv("WORLD_SIZE", "4")
    with pytest.raises(SystemExit) as e:
        bench.main()
    assert "WORLD_SIZE=4" in str(e.value.code)
