"""The bench's reference arm (CPU only: the oracle on this host's cores) keeps
the JSON-line contract: one line, impl = reference, the metric and unit of the
GPU arm, a cpu_baseline describing the run and an e2e object with zero
host<->device bytes."""
import contextlib
import io
import json

import bench


def test_reference_arm_prints_one_contract_line():
    # the default workload (the Llama-3-70B model): each step decodes a
    # sample of it, layer 0's q matrix
    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        rc = bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3"])
    assert rc == 0
    lines = [l for l in out.getvalue().splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "GB/s"
    assert d["higher_is_better"] is True and d["value"] > 0 and d["steps"] == 1 and d["warmup"] == 3
    assert d["config"]["workload"] == "llama3-70b-model-dfloat11"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and "q matrix" in cb["sample"]
    assert "67,108,864 weights" in cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_warmup_below_three_is_refused():
    err = io.StringIO()
    with contextlib.redirect_stderr(err):
        try:
            bench.main(["--warmup", "2"])
        except SystemExit as e:
            assert e.code != 0
        else:
            raise AssertionError("--warmup 2 was accepted")
