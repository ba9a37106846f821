"""bench.py's reference arm (the CPU oracle timed on the host cores), on the CPU.

The arm prints one JSON line on rank 0 with the same metric, unit and workload
config as the GPU arm, plus a cpu_baseline describing the run and an e2e entry
that moves no bytes; under several ranks the other ranks exit 0 silently.
"""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _run(capsys, monkeypatch, rank, world):
    monkeypatch.setenv("RANK", str(rank))
    monkeypatch.setenv("WORLD_SIZE", str(world))
    # the single-thread oracle runs are covered on their own below
    monkeypatch.setattr(bench, "SINGLE_THREAD_RUNS", (("tiny", 2),))
    rc = bench.main(["--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "1",
                     "--gpus", str(world)])
    return rc, capsys.readouterr().out


def test_reference_arm_prints_the_contract_line(capsys, monkeypatch):
    rc, out = _run(capsys, monkeypatch, 0, 1)
    assert rc == 0
    lines = [l for l in out.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["steps"] == 2 and d["warmup"] == 1 and d["n_gpus"] == 1
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["config"] == bench.workload_config("tiny", 1)
    # ms_per_step is the time of the work one step does: all 16 tokens of the tiny batch through its layer
    assert abs(d["value"] - 16 / (d["ms_per_step"] / 1e3)) <= 1e-6 * d["value"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    st = d["cpu_baseline_single_thread"]
    assert [r["workload"] for r in st] == ["tiny"] and st[0]["cores"] == 1 and st[0]["value"] > 0
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


@pytest.mark.parametrize("rank", [1, 3])
def test_reference_arm_other_ranks_exit_quietly(capsys, monkeypatch, rank):
    rc, out = _run(capsys, monkeypatch, rank, 4)
    assert rc == 0 and out.strip() == ""
