"""bench.py's reference arm on CPU: the oracle timed on the host cores, one JSON
line from rank 0 with the same metric as the GPU arm, nothing from other ranks."""
from __future__ import annotations

import contextlib
import io
import json

import bench


def _run(argv, monkeypatch, rank="0", world="1"):
    monkeypatch.setenv("RANK", rank)
    monkeypatch.setenv("LOCAL_RANK", rank)
    monkeypatch.setenv("WORLD_SIZE", world)
    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        rc = bench.main(argv)
    return rc, out.getvalue()


def test_reference_arm_line(monkeypatch):
    rc, text = _run(["--impl", "reference", "--steps", "1", "--warmup", "3", "--cpu-budget", "1"], monkeypatch)
    assert rc == 0
    lines = [l for l in text.splitlines() if l.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference"
    assert line["metric"] == "prefill TFLOP/s (% bf16 TC peak); M=1 GEMV GB/s (% HBM peak)"
    assert line["unit"] == "GB/s" and line["higher_is_better"] is True
    assert line["value"] > 0 and line["steps"] == 1 and line["warmup"] == 3
    assert line["config"] == bench.decode_config(1)           # the GPU arm's config, key for key
    assert line["config"]["workload"] == "q4_0_decode_m1_n12288_k4096" and line["config"]["M"] == 1
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1 and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_print_nothing(monkeypatch):
    rc, text = _run(["--impl", "reference", "--gpus", "2", "--steps", "1"], monkeypatch, rank="1", world="2")
    assert rc == 0 and text == ""
