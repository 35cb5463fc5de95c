"""The benchmark's host-side helpers on CPU: the oracle timing's sample sizes
and thread accounting, and the reference arm's JSON line (the oracle timed on
the host cores, no GPU)."""
import json
import os
import sys
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from diffusion_transformer_joint_jattn_b200 import workloads as W  # noqa: E402


def test_round_heads_multiple_of_workers_capped_at_bh():
    w = W.BY_NAME["t2i_2048_base"]                     # B*H = 48
    assert bench.round_heads(w, 1, 16) == 16
    assert bench.round_heads(w, 17, 16) == 32
    assert bench.round_heads(w, 40.2, 16) == 48
    assert bench.round_heads(w, 100, 16) == 48
    assert bench.round_heads(w, 5, 8) == 8
    tiny = W.BY_NAME["tiny"]                           # B*H = 2
    assert bench.round_heads(tiny, 1, 16) == 2


@pytest.mark.timeout(120)
def test_cpu_baseline_cores_are_the_worker_threads(monkeypatch):
    monkeypatch.setattr(bench.os, "cpu_count", lambda: 2)
    w = W.custom(B=1, H=4, d=64, S_txt=8, grid=8, n_ref=0)
    r = bench.cpu_baseline(w, target_s=0.05)
    assert r["cores"] == 2 and r["blas_threads_per_worker"] == 1 and r["kind"] == "oracle"
    heads = int(r["sample"].split(" heads")[0])
    assert heads % 2 == 0 and 2 <= heads <= w.B * w.H
    assert r["value"] > 0


@pytest.mark.timeout(300)
def test_reference_arm_line(capsys):
    args = types.SimpleNamespace(workload="tiny", steps=1, warmup=1)
    bench.run_reference(args, rank=0, world=1)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["dtype"] == "f64" and line["steps"] == 1
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert line["cpu_baseline"]["cores"] == bench.host_workers()
    assert line["config"]["workload"] == "tiny" and line["value"] > 0


def test_reference_arm_other_ranks_do_nothing(capsys):
    args = types.SimpleNamespace(workload="tiny", steps=1, warmup=1)
    assert bench.run_reference(args, rank=1, world=2) is None
    assert capsys.readouterr().out == ""
