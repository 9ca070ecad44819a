"""The benchmark's reference arm (the FP64 oracle on the host cores) prints the JSON line the
benchmark contract asks for: the same metric, unit and workload as the CUDA arm, its own
CPU-baseline and end-to-end records, and a positive throughput. Runs on the CPU."""
import contextlib
import io
import json

import bench


def test_reference_arm_prints_one_contract_line():
    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        bench.main(["--impl", "reference", "--steps", "1", "--warmup", "0"])
    lines = [ln for ln in out.getvalue().splitlines() if ln.strip().startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "tokens/s"
    assert d["value"] > 0 and d["steps"] == 1 and d["higher_is_better"] is True
    assert d["config"]["workload"].startswith("prefill_bf16_B1_L65536")
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
