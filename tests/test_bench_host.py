"""Host logic of bench.py's roofline reporting (CPU only): the DRAM traffic it
reports comes from a committed ncu capture and only while the captured
kernel's source is unchanged."""
import json
import os

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TRAFFIC = os.path.join(ROOT, "profiles", "traffic.json")


def _records():
    with open(TRAFFIC) as f:
        return {k: v for k, v in json.load(f).items() if not k.startswith("_")}


@pytest.mark.parametrize("kernel", sorted(_records()))
def test_traffic_record_is_complete(kernel):
    rec = _records()[kernel]
    assert os.path.exists(os.path.join(ROOT, "tiled_attention_17_b200", "csrc", rec["source_file"]))
    assert rec["dram_bytes_per_unit"] > 0
    capture = os.path.join(ROOT, rec["capture"])
    assert os.path.exists(capture), f"{kernel}: capture summary {rec['capture']} missing"
    # the summary states the command it came from
    assert "ncu " in open(capture).read()


@pytest.mark.parametrize("kernel", sorted(_records()))
def test_traffic_reported_only_for_the_captured_source(kernel):
    """A record is reported (scaled by the units) while its kernel source is the
    one it was captured from, and as null once that source has changed."""
    rec = _records()[kernel]
    got = bench.recorded_traffic(kernel, rec["source_file"], 2.0)
    if rec["source_sha256_16"] == bench.kernel_source_hash(rec["source_file"]):
        assert got == pytest.approx(2.0 * rec["dram_bytes_per_unit"])
    else:
        assert got is None


def test_stale_or_missing_record_reports_null(monkeypatch):
    rec = _records()["prefill_fwd_kernel"]
    monkeypatch.setattr(bench, "kernel_source_hash", lambda fname: "0" * 16)
    assert bench.recorded_traffic("prefill_fwd_kernel", rec["source_file"], 1.0) is None
    monkeypatch.undo()
    assert bench.recorded_traffic("no_such_kernel", rec["source_file"], 1.0) is None


def test_roofline_fraction():
    r = bench.roofline("tensor", 830.0, 1660.0, "TFLOP/s", None)
    assert r == {"bound": "tensor", "achieved": 830.0, "peak": 1660.0, "unit": "TFLOP/s", "frac": 0.5,
                 "traffic": None}


def test_cpu_baseline_sample_runs_on_host():
    """The CPU-baseline leg (the oracle on a row sample of the causal workload)
    runs on the host alone and states its cores and CPU model."""
    from tiled_attention_17_b200 import inputs
    q, k, v = inputs.prefill_inputs(bench.PREFILL)
    cpu = bench.cpu_oracle_sample(q, k, v, 2048)
    assert cpu["kind"] == "oracle" and cpu["value"] > 0 and cpu["cores"] >= 1
    assert cpu["cpu_model"] and cpu["hardware_threads"] >= 1


def test_cpu_baseline_parity_compares_the_given_output():
    """With the GPU's output given, the CPU-baseline leg reports the parity of
    that output on the rows it evaluated: exact for the oracle's own values,
    failing once one element is off by more than the max-abs bar."""
    import numpy as np

    import oracle
    from tiled_attention_17_b200 import inputs
    c = bench.PREFILL
    q, k, v = inputs.prefill_inputs(c)
    rows, _ = bench.prefill_sample_rows(2048)
    o_ref, lse_ref = oracle.attn(q, k, v, True, scale=c.scale, rows=rows)
    o_full = np.zeros((c.B * c.Hq * c.Nq, c.d))
    lse_full = np.zeros(c.B * c.Hq * c.Nq)
    o_full[rows], lse_full[rows] = o_ref, lse_ref
    par = bench.cpu_oracle_sample(q, k, v, 2048, o_full, lse_full)["parity"]
    assert par["pass"] and par["max_abs"] == 0.0 and par["lse_abs"] == 0.0
    o_full[rows[5], 3] += 0.05
    par = bench.cpu_oracle_sample(q, k, v, 2048, o_full, lse_full)["parity"]
    assert not par["pass"] and abs(par["max_abs"] - 0.05) < 1e-9
