"""The multi-rank plumbing of bench.py (one process per GPU under torchrun) on the host: two gloo
ranks set up the process group from torchrun's environment, run independent layers (distinct
seeds), take the max of their step times over the ranks and agree on the whole-job value; the
reference arm does its work on rank 0 only."""
import os
import socket
import sys
import types

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def rank_main(rank, world, port, out_dir):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import bench
    import gen
    dist, r, n, local = bench.dist_setup(world, backend="gloo")
    assert (r, n, local) == (rank, world, rank) and dist is not None
    w = gen.workload("llama-128k")
    seed = bench.layer_seed(w, r)
    # Each rank's own "step time"; every rank must see the slowest one.
    ms = bench.max_over_ranks(dist, 10.0 + 5.0 * r, torch.device("cpu"))
    seeds = [None] * n
    dist.all_gather_object(seeds, seed)
    dist.barrier()
    value = bench.whole_job_value(w.dense_causal_flops, n, ms)
    with open(os.path.join(out_dir, f"rank{r}.txt"), "w") as f:
        f.write(f"{ms} {value} {len(set(seeds))}\n")
    dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    world = 2
    mp.spawn(rank_main, args=(world, free_port(), str(tmp_path)), nprocs=world, join=True)
    import bench
    import gen
    w = gen.workload("llama-128k")
    rows = [open(tmp_path / f"rank{r}.txt").read().split() for r in range(world)]
    for ms, value, n_seeds in rows:
        assert float(ms) == 15.0  # the max over the two ranks' 10 ms and 15 ms
        assert int(n_seeds) == world  # independent layers
        assert float(value) == pytest.approx(w.dense_causal_flops * world / 15e-3 / 1e12)
    assert rows[0] == rows[1]


def test_single_rank_has_no_process_group(monkeypatch):
    import bench
    for var in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(var, raising=False)
    assert bench.dist_setup(1) == (None, 0, 1, 0)
    assert bench.max_over_ranks(None, 3.5, torch.device("cpu")) == 3.5


def test_reference_arm_other_ranks_do_no_work(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("RANK", "1")
    args = types.SimpleNamespace(workload="llama-128k", tau=0.01, steps=1, warmup=0, gpus=2,
                                 ref_rows=16)
    assert bench.run_reference(args) == 0
    assert capsys.readouterr().out == ""


def test_reference_arm_line_on_rank_0(monkeypatch, capsys):
    """The reference arm (the CPU oracle on a bounded sample) prints one JSON line with the GPU
    arm's metric, unit and config keys, labels its extrapolation and describes its sample."""
    import json

    import bench
    import gen
    for var in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(var, raising=False)
    args = types.SimpleNamespace(workload="tiny", tau=0.01, steps=1, warmup=0, gpus=1, ref_rows=16,
                                 parallel="replica")
    assert bench.run_reference(args) == 0
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["higher_is_better"] is True and d["n_gpus"] == 1 and d["steps"] == 1
    w = gen.workload("tiny", tau=0.01)
    assert d["config"] == bench.workload_config("tiny", w, 1, "replica")
    assert d["value"] > 0 and d["ms_per_step"] > 0
    # A step is the sample itself; the layer's time is the labelled extrapolation of it.
    assert d["layer_ms_extrapolated"] > 0 and "sample" in d["ms_per_step_kind"]
    assert abs(d["value"] - w.dense_causal_flops / (d["layer_ms_extrapolated"] * 1e-3) / 1e12) \
        <= 1e-9 * d["value"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1 and d["cpu_baseline"]["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
