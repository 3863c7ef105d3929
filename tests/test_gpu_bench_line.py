"""bench.py's GPU arm prints the contract line: every key the contract asks for, with
consistent values, on a small decoder-layer step (1024 tokens, 3 timed steps).

Checks the line's own arithmetic (value = GEMM FLOPs / step time, the roofline
fraction = achieved / peak), that every kernel of the step is this library's
(gpu_launches matches the step's launch count), that the clocks were sampled,
and that the CPU baseline is the oracle's."""
import json

import pytest

import bench
from tests.gpu_helpers import require_cuda

pytestmark = pytest.mark.gpu


def test_gpu_arm_prints_the_contract_line(capsys, monkeypatch):
    require_cuda()
    monkeypatch.delenv("RANK", raising=False)
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    assert bench.main(["--tokens", "1024", "--steps", "3", "--warmup", "3", "--no-extra"]) == 0
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.strip().startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["metric"] == bench.METRIC and d["unit"] == "TFLOP/s"
    assert (d["n_gpus"], d["steps"], d["warmup"]) == (1, 3, 3)
    assert d["higher_is_better"] is True and d["scaling"] == "weak" and d["vs_baseline"] is None
    assert d["dtype"] == "e4m3" and d["data"] == "synthetic"
    assert d["config"]["tokens_per_gpu"] == 1024 and "flushed" in d["config"]["l2"]
    flops = sum(2 * 1024 * n * k * 3 for _, n, k in bench.workloads.LAYER_GEMMS)
    assert d["value"] == pytest.approx(flops / (d["ms_per_step"] * 1e-3) / 1e12, rel=1e-6)
    r = d["roofline"]
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["peak"] > 0
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"], rel=1e-9)
    assert r["traffic"] is None            # the captured traffic is that of the 16384-token step
    q = d["quant"]
    assert q["frac"] == pytest.approx(q["achieved_gbs"] / q["peak_gbs"], rel=1e-9)
    e = d["e2e"]
    assert e["unit"] == "TFLOP/s" and 0 < e["value"] < d["value"]
    assert e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    cpu = d["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["cores"] >= 1 and cpu["value"] > 0 and cpu["sample"]
    c = d["clocks"]
    assert c["samples"] >= 1 and c["sm_mhz"] > 0 and c["sm_max_mhz"] > 0 and isinstance(c["reasons"], list)
    ops = d["per_op_median"]
    assert "weights.quant_w" in ops and len([k for k in ops if "gemm" in k]) == 12
    launches = sum(2 if v.get("split_k", 1) > 1 else 1 for v in ops.values())
    assert d["gpu_launches"] == launches * 3
    assert d["device_error"] == "FP8BLK_OK"
