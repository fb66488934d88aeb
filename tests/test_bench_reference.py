"""bench.py's reference arm (the CPU oracle) on small samples: it prints one
JSON line with the benchmark contract's keys, and ranks other than 0 print
nothing. Runs on CPU only (no GPU, no CUDA library needed)."""
import contextlib
import io
import json

import pytest

import bench

REQUIRED = ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
            "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e")


def _run(argv):
    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        rc = bench.main(argv)
    return rc, [ln for ln in out.getvalue().splitlines() if ln.strip()]


@pytest.mark.parametrize("workload,rows", [("tiny", 4), ("polar", 2), ("decode_13b", 1), ("stack_1p1b", 1), ("decode_gemm", 1)])
def test_reference_arm_prints_one_contract_line(monkeypatch, workload, rows):
    monkeypatch.delenv("RANK", raising=False)
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    rc, lines = _run(["--impl", "reference", "--workload", workload, "--steps", "1", "--warmup", "0",
                      "--cpu-rows", str(rows)])
    assert rc == 0 and len(lines) == 1
    d = json.loads(lines[0])
    for k in REQUIRED:
        assert k in d, k
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert "workload" in d["config"]


def test_reference_arm_other_ranks_print_nothing(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    rc, lines = _run(["--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "0"])
    assert rc == 0 and lines == []
