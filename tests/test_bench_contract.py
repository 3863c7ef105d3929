"""bench.py's command-line contract, checked on the CPU.

The reference arm (the oracle timed on the host cores) runs without a GPU, so
its JSON line is checked here key by key; the GPU arm's line is produced by
the same keys and is exercised on the GPU machine.  Also: ranks other than 0 of a
multi-process reference run print nothing, and fewer than three warm-up steps
are refused.
"""
import json

import pytest

import bench


def _one_json_line(text):
    lines = [ln for ln in text.splitlines() if ln.strip().startswith("{")]
    assert len(lines) == 1, text
    return json.loads(lines[0])


def test_reference_arm_prints_the_contract_line(capsys, monkeypatch):
    monkeypatch.delenv("RANK", raising=False)
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3", "--workload", "qkv_fwd"]) == 0
    line = _one_json_line(capsys.readouterr().out)
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["unit"] == "TFLOP/s"
    assert line["value"] > 0 and line["ms_per_step"] > 0
    assert (line["n_gpus"], line["steps"], line["warmup"]) == (1, 1, 3)
    assert line["higher_is_better"] is True and line["scaling"] == "weak" and line["vs_baseline"] is None
    assert line["dtype"] == "f64" and line["data"] == "synthetic"
    assert line["config"]["workload"] == bench.WORKLOAD_DESC["qkv_fwd"]
    cpu = line["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["value"] == line["value"] and cpu["cores"] >= 1 and cpu["sample"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_print_nothing(capsys, monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]) == 0
    assert capsys.readouterr().out.strip() == ""


def test_fewer_than_three_warmup_steps_are_refused(monkeypatch):
    monkeypatch.delenv("RANK", raising=False)
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    with pytest.raises(SystemExit):
        bench.main(["--impl", "reference", "--steps", "1", "--warmup", "2"])


def test_gpu_count_must_match_the_launch(monkeypatch):
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    with pytest.raises(SystemExit):
        bench.main(["--gpus", "2", "--steps", "1", "--warmup", "3"])
